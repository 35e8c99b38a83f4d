"""Benchmark of the DiT joint-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload flux_2048] [--impl ours|reference]
                    [--mode replicas|ring|ring_peers|ulysses|ulysses_peers]

One step = one pass of the whole hot path over one batch of synthetic input of the chosen
workload (default: FLUX-2048-like joint attention, B=1 H=24 S=16896 D=128, bf16):
    1. dit_attn_fwd         full attention forward (out bf16 + lse)
    2. dit_attn_fwd_chunk   x n_chunks: the same queries against n equal KV chunks (fp32 partials)
    3. dit_attn_merge       exact LSE merge of the n partials (bf16 out + lse)
For the video workload the FP8 variant adds dit_quant_fp8 of Q, K, V and an E4M3 forward.

Metric: TFLOP/s counted as 4*B*H*S^2*D per attention pass (the full pass and the chunked
pass each count once), whole job, max over ranks.  Inputs (Q, K, V) are resident in HBM and
larger than the 126 MB L2, so no L2 flush is needed between steps.  Multi-GPU (torchrun):
every rank runs its own replica batch (independent problems; no data-path collective),
scaling "weak".

--mode ring|ring_peers|ulysses|ulysses_peers instead splits ONE sequence of the workload
across the ranks by a sequence-parallel form of the xDiT overview page (section 3.2.2): the
KV ring over NCCL with fused ring steps, the ring without a ring over peer memory, the
Ulysses all-to-all over NCCL, or Ulysses fused over peer memory.  A step is one attention over
the whole sequence; value = its FLOPs / max-over-ranks time, scaling "strong".

--impl reference times the fp64 CPU oracle (the only other implementation of this path) on
the host cores, on a bounded sample of the same workload per step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import WORKLOADS, chunk_bounds, make_qkv  # noqa: E402

METRIC = "DiT attention TFLOP/s (4·B·H·S²·D) and % of B200 dense BF16/FP8 peak, 1 GPU"
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_fwd_bf16_flux2048.txt")
KERNEL_SRC = os.path.join(ROOT, "long_sequence_attention_b200", "csrc", "attn_fwd.cuh")
# used only when MEASURED_PEAKS.json is absent: an earlier B200 measurement (HBM
# copy, burst cuBLAS bf16); there is no fallback for the sustained figure
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ----------------------------------------------------------------------------- helpers
def rank_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def replica_seed_offset(rank: int) -> int:
    """Each rank runs its own replica batch: the workload seeds shift by 10 per rank."""
    return 10 * rank


class Ranks:
    """Process-group plumbing of a multi-rank run: every rank makes the same calls in the
    same order; timing is reduced to the max over ranks.  With world == 1 it is a no-op."""

    def __init__(self, world: int, backend: str = "nccl", device=None, timeout_s: int = 120):
        self.world, self.backend, self.device, self.timeout_s = world, backend, device, timeout_s

    def init(self):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": self.device} if (self.backend == "nccl" and self.device is not None) else {}
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=self.timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        if self.world == 1:
            return float(x)
        import torch
        import torch.distributed as dist
        dev = self.device if self.backend == "nccl" else "cpu"
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_hash() -> str:
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the full-forward kernel from the committed ncu summary, or
    None when there is none or the kernel source changed since it was captured."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    vals = {}
    with open(PROFILE_SUMMARY) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != kernel_hash():
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def smi_device_id(dev) -> str:
    """nvidia-smi -i argument for a torch device (its UUID, immune to CUDA_VISIBLE_DEVICES)."""
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(dev.index or 0)


REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """SM clock and throttle-reason samples during the timed region: through NVML every 10 ms
    when the bindings load (reading only; nothing is set), else nvidia-smi every 100 ms."""

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.nvml = None
        self.stop = threading.Event()

    def _nvml_sample(self, nv, handle):
        sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
        mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
        self.lines.append(f"{sm}, {mx}, 0, {bits:#x}")

    def _nvml_loop(self, nv, handle):
        while not self.stop.is_set():
            try:
                self._nvml_sample(nv, handle)
            except Exception:
                return
            self.stop.wait(0.01)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            dev = str(self.dev)
            handle = (nv.nvmlDeviceGetHandleByUUID(dev) if dev.startswith("GPU-")
                      else nv.nvmlDeviceGetHandleByIndex(int(dev)))
            self.nvml = nv
            self.handle = handle
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, handle), daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 2.0:
                time.sleep(0.005)
            self.lines.clear()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.02)         # sampler is up before the timed region starts
            self.lines.clear()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.nvml is not None:
            self.stop.set()
            self.thread.join(timeout=2)
            try:
                self._nvml_sample(self.nvml, self.handle)   # one at the end: short regions get one too
            except Exception:
                pass
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 4:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                bits = int(parts[3], 16) if parts[3].startswith("0x") else int(parts[3])
            except ValueError:
                continue
            for b, name in REASON_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvml, 10 ms" if self.nvml is not None else "nvidia-smi, 100 ms"}


# ----------------------------------------------------------------------------- our arm
class Step:
    """Device buffers and the launch sequence of one step of the hot path."""

    def __init__(self, lsa, w, data, dev, fp8: bool):
        import torch
        self.lsa, self.w, self.fp8 = lsa, w, fp8
        B, H, S, D = w.B, w.H, w.S, w.D
        to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        self.q, self.k, self.v = (to_dev(data[n + "_bits"]) for n in "qkv")
        self.out = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
        self.bounds = chunk_bounds(S, w.n_chunks) if w.n_chunks > 1 else []
        self.parts = [(torch.empty((B, H, S, D), dtype=torch.float32, device=dev),
                       torch.empty((B, H, S), dtype=torch.float32, device=dev)) for _ in self.bounds]
        self.mout = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=dev)
        self.mlse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
        if fp8:
            n = B * H * S * D
            self.codes = [torch.empty((B, H, S, D), dtype=torch.uint8, device=dev) for _ in range(3)]
            self.descale = torch.empty((3,), dtype=torch.float32, device=dev)
            self.ws_bytes = lsa.dit_quant_fp8_workspace_bytes(n)
            self.ws = torch.empty((self.ws_bytes // 4,), dtype=torch.float32, device=dev)
            self.out8 = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=dev)
            self.lse8 = torch.empty((B, H, S), dtype=torch.float32, device=dev)

    @property
    def launches(self) -> int:
        n = 1
        if self.bounds:
            n += len(self.bounds) + 1
        if self.fp8:
            n += 3 * 2 + 1
        return n

    @property
    def flops(self) -> float:
        f = self.w.flops * (1 + (1 if self.bounds else 0))
        if self.fp8:
            f += self.w.flops
        return f

    def run_heads(self, stream, g0: int, g1: int):
        """The bf16 part of the step (full forward, chunks, merge) on the flattened heads
        [g0, g1) of [B*H, S, D]: heads are independent, so a slice is a valid call with B = 1
        and H = g1 - g0 on offset pointers."""
        lsa, w = self.lsa, self.w
        S, D, n = w.S, w.D, g1 - g0

        def sl(t, per_row):
            return t.data_ptr() + g0 * S * per_row * t.element_size()
        q, k, v = sl(self.q, D), sl(self.k, D), sl(self.v, D)
        lsa.dit_attn_fwd(q, k, v, sl(self.out, D), sl(self.lse, 1), 1, n, S, D, w.scale, lsa.DIT_BF16, None, stream)
        for (a, b), (po, pl) in zip(self.bounds, self.parts):
            lsa.dit_attn_fwd_chunk(q, k, v, sl(po, D), sl(pl, 1), 1, n, S, S, D, a, b, w.scale, lsa.DIT_BF16,
                                   lsa.DIT_FP32, None, stream)
        if self.bounds:
            lsa.dit_attn_merge([sl(p[0], D) for p in self.parts], [sl(p[1], 1) for p in self.parts],
                               sl(self.mout, D), sl(self.mlse, 1), 1, n, S, D, lsa.DIT_FP32, lsa.DIT_BF16, stream)

    def run(self, stream, ev=None):
        lsa, w = self.lsa, self.w
        B, H, S, D = w.B, w.H, w.S, w.D
        if ev is not None:
            ev[0].record(stream)
        lsa.dit_attn_fwd(self.q, self.k, self.v, self.out, self.lse, B, H, S, D, w.scale, lsa.DIT_BF16, None, stream)
        if ev is not None:
            ev[1].record(stream)
        for (a, b), (po, pl) in zip(self.bounds, self.parts):
            lsa.dit_attn_fwd_chunk(self.q, self.k, self.v, po, pl, B, H, S, S, D, a, b, w.scale, lsa.DIT_BF16,
                                   lsa.DIT_FP32, None, stream)
        if self.bounds:
            if ev is not None:
                ev[2].record(stream)
            lsa.dit_attn_merge([p[0] for p in self.parts], [p[1] for p in self.parts], self.mout, self.mlse,
                               B, H, S, D, lsa.DIT_FP32, lsa.DIT_BF16, stream)
            if ev is not None:
                ev[3].record(stream)
        self.run_fp8(stream, ev)

    def run_fp8(self, stream, ev=None):
        lsa, w = self.lsa, self.w
        B, H, S, D = w.B, w.H, w.S, w.D
        if self.fp8:
            n = B * H * S * D
            for i, x in enumerate((self.q, self.k, self.v)):
                lsa.dit_quant_fp8(x, self.codes[i], self.descale[i:i + 1], n, self.ws, self.ws_bytes, stream)
            if ev is not None:
                ev[4].record(stream)
            lsa.dit_attn_fwd(self.codes[0], self.codes[1], self.codes[2], self.out8, self.lse8, B, H, S, D,
                             w.scale, lsa.DIT_FP8_E4M3, self.descale, stream)
            if ev is not None:
                ev[5].record(stream)


SEQPAR_MODES = ("ring", "ring_peers", "ulysses", "ulysses_peers")


def seqpar_blocks(mode: str, S: int, H: int, P: int):
    """Rows [a, b) of the sequence each of P ranks holds in a sequence-parallel mode, or a
    one-line reason why the split is not supported.  The NCCL ring takes any split (the last
    rank gets the remainder); the peer-memory ring and both Ulysses forms need S/P rows per
    rank, a multiple of 128 when P > 1 (a 128-row tile must not straddle two ranks), and
    Ulysses needs H divisible by P."""
    if mode == "ring":
        return chunk_bounds(S, P), None
    if S % P != 0 or (P > 1 and (S // P) % 128 != 0):
        return None, f"{mode} needs S/P rows per rank, a multiple of 128 (S={S}, P={P})"
    if mode in ("ulysses", "ulysses_peers") and H % P != 0:
        return None, f"{mode} needs H divisible by P (H={H}, P={P})"
    if mode in ("ring_peers", "ulysses_peers") and P > 8:
        return None, f"{mode} reads at most 8 ranks' blocks"
    n = S // P
    return [(r * n, (r + 1) * n) for r in range(P)], None


def seqpar_launches(mode: str, B: int, P: int) -> int:
    """Library kernel launches of one sequence-parallel step on one rank."""
    if mode == "ring":
        return 1 + P + 1                    # accumulator init, P fused ring steps, bf16 finish
    if mode == "ulysses":
        return 1 + (5 if (B > 1 and P > 1) else 0)   # attention (+ layout swaps at B > 1)
    return 1                                # one fused multi-block launch


def run_seqpar(args, rank, local_rank, world):
    """One attention over the workload's whole sequence, split across the ranks by a USP
    dimension (xDiT overview, section 3.2.2): each rank holds a block of rows of Q, K, V and
    gets its rows of O and LSE.  value = the one attention's FLOPs per step / max-over-ranks
    time (strong scaling: the total work is fixed as ranks are added)."""
    import datetime
    import torch
    import torch.distributed as dist
    if rank == 0 or world == 1:
        ensure_library()
    if world > 1:
        deadline = time.time() + 900
        lib = os.path.join(ROOT, "long_sequence_attention_b200", "libdit_attn.so")
        while not os.path.exists(lib) and time.time() < deadline:
            time.sleep(1.0)
    import long_sequence_attention_b200 as lsa
    from long_sequence_attention_b200 import ring as lring
    from long_sequence_attention_b200 import ulysses as lul

    w = WORKLOADS[args.workload]
    B, H, S, D = w.B, w.H, w.S, w.D
    blocks, why = seqpar_blocks(args.mode, S, H, world)
    if why is not None:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "mode": args.mode, "n_gpus": world, "unavailable": why}), flush=True)
        return
    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    else:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
        dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    ranks = Ranks(world, "nccl", dev)

    data = make_qkv(w)                      # one sequence, the same on every rank; each keeps its rows
    a, b = blocks[rank]
    to_dev = lambda name: torch.from_numpy(np.ascontiguousarray(data[name + "_bits"][:, :, a:b]).view(np.int16)) \
        .view(torch.bfloat16).to(dev)
    q, k, v = to_dev("q"), to_dev("k"), to_dev("v")
    peer_ops = lul.CudaPeerOps() if args.mode in ("ring_peers", "ulysses_peers") else None
    out_buf = torch.empty_like(q)
    lse_buf = torch.empty((B, H, b - a), dtype=torch.float32, device=dev)

    def step():
        if args.mode == "ring":
            return lring.ring_attention_dist(q, k, v, w.scale, out_dtype=torch.bfloat16, block_lens=[y - x for x, y in blocks])
        if args.mode == "ring_peers":
            return lring.ring_attention_peers(q, k, v, w.scale, ops=peer_ops, out=out_buf, lse=lse_buf)
        if args.mode == "ulysses":
            return lul.ulysses_attention_dist(q, k, v, w.scale)
        return lul.ulysses_attention_peers(q, k, v, w.scale, ops=peer_ops, out=out_buf, lse=lse_buf)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if lsa.dit_device_status(clear=True) != 0:
        raise RuntimeError("device status after warm-up is not OK")
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(smi_device_id(dev)) as clk:
        t0.record()
        for _ in range(args.steps):
            o, l = step()
        t1.record()
        torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    elapsed_ms = ranks.max(t0.elapsed_time(t1))
    status = lsa.dit_device_status(clear=True)

    # this rank's rows against a local forward over the whole sequence (one launch)
    kf, vf = (torch.from_numpy(data[n + "_bits"].view(np.int16)).view(torch.bfloat16).to(dev) for n in "kv")
    ref_o = torch.empty((B, H, b - a, D), dtype=torch.float32, device=dev)
    ref_l = torch.empty((B, H, b - a), dtype=torch.float32, device=dev)
    qs = q.contiguous()
    lsa.dit_attn_fwd_chunk(qs, kf, vf, ref_o, ref_l, B, H, b - a, S, D, 0, S, w.scale, lsa.DIT_BF16, lsa.DIT_FP32)
    torch.cuda.synchronize()
    diff = ranks.max(float((o.float() - ref_o).abs().max().item()))
    ldiff = ranks.max(float((l - ref_l).abs().max().item()))
    del kf, vf, ref_o, ref_l

    # end to end: this rank's rows copied in from pinned host memory and its O/LSE copied back
    host_in = [torch.from_numpy(np.ascontiguousarray(data[n + "_bits"][:, :, a:b]).view(np.int16))
               .view(torch.bfloat16).pin_memory() for n in "qkv"]
    host_o = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    host_l = torch.empty((B, H, b - a), dtype=torch.float32).pin_memory()
    n_e2e = max(3, min(args.steps, 10))

    def e2e_step():
        for h, d_ in zip(host_in, (q, k, v)):
            d_.copy_(h, non_blocking=True)
        o_, l_ = step()
        host_o.copy_(o_, non_blocking=True)
        host_l.copy_(l_, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = ranks.max(e0.elapsed_time(e1)) / n_e2e
    if peer_ops is not None:
        dist.barrier()
        peer_ops.close()
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return
    peaks, peaks_src = load_peaks()
    ms = elapsed_ms / args.steps
    value = w.flops / (ms * 1e-3) / 1e12
    per_gpu = value / world
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) rounded to bf16; no weights involved)",
        "config": {"workload": w.name, "B": B, "H": H, "S": S, "D": D, "scale": w.scale,
                   "step": {"ring": "ring_attention_dist (NCCL send/recv + dit_attn_fwd_chunk_acc)",
                            "ring_peers": "ring_attention_peers (dit_attn_fwd_parts over peer memory)",
                            "ulysses": "ulysses_attention_dist (NCCL all-to-all + dit_attn_fwd_seg)",
                            "ulysses_peers": "ulysses_attention_peers (dit_attn_fwd_parts over peer memory)"}[args.mode],
                   "rows_per_rank": [y - x for x, y in blocks],
                   "l2": "no flush: Q/K/V exceed the 126 MB L2" if 3 * B * H * S * D * 2 > 126e6 else "inputs fit in L2",
                   "parallelism": f"{args.mode}{world}"},
        "roofline": {"bound": "tensor", "kernel": args.mode + " step, per GPU", "achieved": round(per_gpu, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(per_gpu / peaks["bf16_tflops"], 4),
                     "peak_source": f"{peaks_src} bf16_tflops (burst)", "traffic": None},
        "gpu_launches": seqpar_launches(args.mode, B, world) * args.steps,
        "device_status": status,
        "max_abs_vs_single_launch": diff, "lse_max_abs_vs_single_launch": ldiff,
        "clocks": clk.summary(),
        "e2e": {"value": round(w.flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 3),
                "steps": n_e2e, "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in host_in) * world,
                "d2h_bytes_per_step": (host_o.numel() * 2 + host_l.numel() * 4) * world},
    }
    if world == 1 and not args.skip_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def ensure_library():
    """Build the in-tree CUDA library if it is missing or older than its sources (a no-op
    otherwise), without importing the package first."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_lsa_build", os.path.join(ROOT, "long_sequence_attention_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def run_ours(args, rank, local_rank, world):
    import torch
    if rank == 0 or world == 1:
        ensure_library()
    if world > 1:
        # other ranks wait for rank 0's build through the file system: the library appears
        # (os.replace) only when complete
        deadline = time.time() + 900
        lib = os.path.join(ROOT, "long_sequence_attention_b200", "libdit_attn.so")
        while not os.path.exists(lib) and time.time() < deadline:
            time.sleep(1.0)
    import long_sequence_attention_b200 as lsa

    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    ranks = Ranks(world, "nccl", dev)
    ranks.init()
    w = WORKLOADS[args.workload]
    fp8 = args.workload == "video"
    data = make_qkv(w, seed_offset=replica_seed_offset(rank))   # each rank: its own replica batch
    stream = torch.cuda.Stream(device=dev)
    step = Step(lsa, w, data, dev, fp8)
    barrier = ranks.barrier

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step.run(stream)
    stream.synchronize()
    if lsa.dit_device_status(clear=True) != 0:
        raise RuntimeError("device status after warm-up is not OK")

    n_ev = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(smi_device_id(dev)) as clk:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(args.steps):
                step.run(stream, evs[i])
            t1.record(stream)
        stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    elapsed_ms = ranks.max(t0.elapsed_time(t1))
    status = lsa.dit_device_status(clear=True)

    full_ms = [e[0].elapsed_time(e[1]) for e in evs]
    chunk_ms = [e[1].elapsed_time(e[2]) for e in evs] if step.bounds else []
    merge_ms = [e[2].elapsed_time(e[3]) for e in evs] if step.bounds else []
    fp8_ms = [e[4].elapsed_time(e[5]) for e in evs] if fp8 else []

    # end to end through the C ABI with host buffers: pinned H2D of Q, K, V, the step, D2H of
    # the outputs, all inside the timed region
    e2e = run_e2e(args, lsa, step, data, stream, dev, ranks)
    ring = run_ring_fused(lsa, step, stream, ranks) if step.bounds else None
    na = run_na3d_context(lsa, dev, stream, ranks)
    seg = run_seg_context(lsa, step, stream, ranks)
    parts = run_parts_context(lsa, step, stream, ranks)
    fp8b = run_fp8_blocks_context(lsa, step, stream, ranks)
    fwds = run_forwards_context(lsa, dev, stream, ranks) if not args.skip_forwards else None

    ranks.close()
    if rank != 0:
        return

    peaks, peaks_src = load_peaks()
    total_flops = step.flops * args.steps * world
    value = total_flops / (elapsed_ms * 1e-3) / 1e12
    avg_full = statistics.mean(full_ms)
    achieved = w.flops / (avg_full * 1e-3) / 1e12
    # Denominator: the burst cuBLAS figure for a kernel timed alone, the sustained one (seconds
    # of back-to-back GEMMs under the power cap) when the kernel runs inside a timed region of
    # a second or more of continuous work, as here with the default step count.
    long_region = elapsed_ms >= 1000.0 and "bf16_tflops_sustained" in peaks
    peak = peaks["bf16_tflops_sustained"] if long_region else peaks["bf16_tflops"]
    peak_src = (f"{peaks_src} bf16_tflops_sustained (kernel timed inside {elapsed_ms / 1000:.1f} s of "
                f"back-to-back steps)" if long_region else f"{peaks_src} bf16_tflops (burst)")
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) rounded to bf16; no weights involved)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "D": w.D, "scale": w.scale,
                   "n_chunks": w.n_chunks, "fp8_variant": fp8,
                   "step": "dit_attn_fwd" + (" + %d x dit_attn_fwd_chunk + dit_attn_merge" % len(step.bounds)
                                             if step.bounds else "")
                           + (" + 3 x dit_quant_fp8 + dit_attn_fwd(e4m3)" if fp8 else ""),
                   "l2": "no flush: Q/K/V (%.0f MB) exceed the 126 MB L2" % (3 * w.B * w.H * w.S * w.D * 2 / 1e6),
                   "parallelism": "replicas%d" % world},
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel<128,bf16> (dit_attn_fwd)",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_src,
                     "frac_of_burst": round(achieved / peaks["bf16_tflops"], 4),
                     "frac_of_sustained": round(achieved / peaks.get("bf16_tflops_sustained", peak), 4),
                     "traffic": profiled_traffic(),
                     "algorithmic_bytes": 4 * w.B * w.H * w.S * w.D * 2 + w.B * w.H * w.S * 4},
        "phases_ms": {"full_fwd": round(avg_full, 4),
                      "chunks": round(statistics.mean(chunk_ms), 4) if chunk_ms else None,
                      "merge": round(statistics.mean(merge_ms), 4) if merge_ms else None,
                      "fp8_fwd": round(statistics.mean(fp8_ms), 4) if fp8_ms else None},
        "gpu_launches": step.launches * args.steps,
        "device_status": status,
    }
    if merge_ms:
        n = len(step.bounds)
        mbytes = (n * (w.B * w.H * w.S * (w.D * 4 + 4)) + w.B * w.H * w.S * (w.D * 2 + 4))
        gbs = mbytes / (statistics.mean(merge_ms) * 1e-3) / 1e9
        line["merge_roofline"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                                  "algorithmic_bytes": mbytes}
    if fp8_ms:
        line["fp8_fwd_tflops"] = round(w.flops / (statistics.mean(fp8_ms) * 1e-3) / 1e12, 2)
    if ring is not None:
        ring["chunks_plus_merge_ms"] = round((statistics.mean(chunk_ms) + statistics.mean(merge_ms)), 4)
        line["ring_fused"] = ring
    line["na3d"] = na
    if seg is not None:
        line["ulysses_seg"] = seg
    if parts is not None:
        line["ulysses_peers_virtual"] = parts
    line["fp8_blocks"] = fp8b
    if fwds is not None:
        line["forwards"] = fwds
    line["clocks"] = clk.summary()
    line["e2e"] = e2e
    if world == 1 and not args.skip_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_na3d_context(lsa, dev, stream, ranks, reps: int = 10):
    """3-D neighborhood attention on the video token grid (21 x 30 x 52, 40 heads, D = 128,
    7 x 7 x 7 window), reported beside the step: its own kernel time, useful FLOP/s (keys in
    windows) and executed FLOP/s (visited tiles).  Inputs are drawn on the device: this is a
    kernel timing; parity is covered by the tests."""
    import torch
    grid, kernel, H, D = (21, 30, 52), (7, 7, 7), 40, 128
    S = grid[0] * grid[1] * grid[2]
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    q, k, v = (torch.randn((1, H, S, D), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
               for _ in range(3))
    out = torch.empty_like(q)
    lse = torch.empty((1, H, S), dtype=torch.float32, device=dev)
    call = lambda: lsa.dit_na3d_fwd(q, k, v, out, lse, 1, H, *grid, D, *kernel, D ** -0.5, stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
        stream.synchronize()
        ranks.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            call()
        t1.record(stream)
    stream.synchronize()
    ms = ranks.max(t0.elapsed_time(t1)) / reps
    useful = 4.0 * H * S * kernel[0] * kernel[1] * kernel[2] * D
    plan = lsa.dit_na3d_plan(*grid, *kernel)           # the kernel's own tiling (host call)
    executed = 4.0 * H * plan["steps_per_head"] * 256 * 128 * D
    del q, k, v, out, lse
    return {"grid": list(grid), "window": list(kernel), "heads": H, "D": D, "ms": round(ms, 4),
            "useful_tflops": round(useful * ranks.world / (ms * 1e-3) / 1e12, 2),
            "executed_tflops": round(executed * ranks.world / (ms * 1e-3) / 1e12, 2),
            "tile_efficiency": round(useful / executed, 4), "q_brick": list(plan["q_brick"]),
            "steps_per_head": plan["steps_per_head"], "call": "dit_na3d_fwd"}


def _time_calls(call, stream, ranks, reps: int = 10) -> float:
    """ms per call: CUDA events on the launching stream after 3 warm-up calls, max over ranks."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
        stream.synchronize()
        ranks.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            call()
        t1.record(stream)
    stream.synchronize()
    return ranks.max(t0.elapsed_time(t1)) / reps


def run_seg_context(lsa, step, stream, ranks):
    """dit_attn_fwd_seg on the step's Q/K/V laid out as a 4-way sequence all-to-all delivers
    them ([4, B*H, S/4, D]), beside dit_attn_fwd on the plain layout: the segmented
    addressing of the Ulysses path should cost nothing."""
    import torch
    w = step.w
    B, H, S, D = w.B, w.H, w.S, w.D
    P = 4
    if S % P or (S // P) % 128:
        return None
    seg = S // P
    lay = lambda x: x.reshape(B * H, P, seg, D).transpose(0, 1).contiguous()
    q, k, v = lay(step.q), lay(step.k), lay(step.v)
    out = torch.empty_like(q)
    lse = torch.empty((P, B * H, seg), dtype=torch.float32, device=q.device)
    ms_seg = _time_calls(lambda: lsa.dit_attn_fwd_seg(q, k, v, out, lse, B, H, S, D, seg, w.scale, lsa.DIT_BF16,
                                                      lsa.DIT_BF16, None, stream), stream, ranks)
    ms_plain = _time_calls(lambda: lsa.dit_attn_fwd(step.q, step.k, step.v, step.out, step.lse, B, H, S, D, w.scale,
                                                    lsa.DIT_BF16, None, stream), stream, ranks)
    same = bool(torch.equal(out.transpose(0, 1).reshape(B, H, S, D), step.out))
    del q, k, v, out, lse
    return {"segments": P, "seg_rows": seg, "ms": round(ms_seg, 4), "plain_layout_ms": round(ms_plain, 4),
            "tflops": round(w.flops * ranks.world / (ms_seg * 1e-3) / 1e12, 2),
            "bit_identical_to_plain": same, "call": "dit_attn_fwd_seg"}


def run_parts_context(lsa, step, stream, ranks):
    """dit_attn_fwd_parts as 4 ranks would run it (each rank's rows in its own buffers, one
    launch per rank for a quarter of the heads), here as 4 launches one after another on this
    GPU: the fused Ulysses step's kernel time with all blocks local."""
    import torch
    w = step.w
    B, H, S, D = w.B, w.H, w.S, w.D
    P = 4
    if S % P or (S // P) % 128 or H % P:
        return None
    rows = S // P
    blocks = [[x[:, :, r * rows:(r + 1) * rows].contiguous() for x in (step.q, step.k, step.v)] for r in range(P)]
    outs = [torch.empty((B, H, rows, D), dtype=torch.bfloat16, device=step.q.device) for _ in range(P)]
    lses = [torch.empty((B, H, rows), dtype=torch.float32, device=step.q.device) for _ in range(P)]

    def call():
        for r in range(P):
            lsa.dit_attn_fwd_parts([b[0] for b in blocks], [b[1] for b in blocks], [b[2] for b in blocks], outs, lses,
                                   B, H, r * (H // P), H // P, rows, D, w.scale, stream)
    ms = _time_calls(call, stream, ranks)
    full = torch.cat(outs, dim=2)
    same = bool(torch.equal(full, step.out))
    del blocks, outs, lses, full
    return {"ranks": P, "ms_all_launches": round(ms, 4), "tflops": round(w.flops * ranks.world / (ms * 1e-3) / 1e12, 2),
            "bit_identical_to_plain": same, "call": "4 x dit_attn_fwd_parts (virtual ranks, blocks local)"}


def run_fp8_blocks_context(lsa, step, stream, ranks):
    """Per-block E4M3 on the step's Q/K/V: dit_quant_fp8_blocks of the three tensors (HBM-bound)
    and dit_attn_fwd_fp8_blocks (against 2x the measured bf16 peak, the nominal e4m3 ratio)."""
    import torch
    w = step.w
    B, H, S, D = w.B, w.H, w.S, w.D
    if D != 128:
        return None
    nb = (S + 127) // 128
    codes = [torch.empty((B, H, S, D), dtype=torch.uint8, device=step.q.device) for _ in range(3)]
    ds = [torch.empty((B, H, nb), dtype=torch.float32, device=step.q.device) for _ in range(3)]
    out = torch.empty_like(step.out)
    lse = torch.empty_like(step.lse)

    def quant():
        for x, c, d in zip((step.q, step.k, step.v), codes, ds):
            lsa.dit_quant_fp8_blocks(x, c, d, B, H, S, D, stream)
    ms_q = _time_calls(quant, stream, ranks)
    ms_f = _time_calls(lambda: lsa.dit_attn_fwd_fp8_blocks(*codes, *ds, out, lse, B, H, S, S, D, 0, S, w.scale,
                                                          lsa.DIT_BF16, stream), stream, ranks)
    peaks, _ = load_peaks()
    tf = w.flops * ranks.world / (ms_f * 1e-3) / 1e12
    qbytes = 3 * B * H * S * D * 3 + 3 * B * H * nb * 4
    del codes, ds, out, lse
    return {"quant_ms_3_tensors": round(ms_q, 4), "quant_gbs": round(qbytes / (ms_q * 1e-3) / 1e9, 1),
            "fwd_ms": round(ms_f, 4), "fwd_tflops": round(tf, 2),
            "fwd_frac_of_2x_bf16_peak": round(tf / (2 * peaks["bf16_tflops"]), 4),
            "calls": "3 x dit_quant_fp8_blocks, dit_attn_fwd_fp8_blocks"}


def run_forwards_context(lsa, dev, stream, ranks, reps: int = 5):
    """The forward kernel alone on every DiT workload of the suite, beside the step: bf16 on
    SD3-1024 (D = 64), FLUX-1024, FLUX-2048 and video, and E4M3 with per-tensor scales on
    FLUX-2048 and video.  Inputs are N(0,1) drawn on the device (timing only; parity of every
    configuration is covered by the tests).  bf16 against the measured bf16 peak, E4M3 against
    twice it (the nominal dense FP8 / BF16 ratio)."""
    import torch
    peaks, src = load_peaks()
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    res = {}
    plan = [("sd3_1024", False), ("flux_1024", False), ("flux_2048", False), ("video", False),
            ("flux_2048", True), ("video", True)]
    for name, fp8 in plan:
        w = WORKLOADS[name]
        B, H, S, D = w.B, w.H, w.S, w.D
        x = [torch.randn((B, H, S, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(3)]
        out = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
        if fp8:
            n = B * H * S * D
            codes = [torch.empty((B, H, S, D), dtype=torch.uint8, device=dev) for _ in range(3)]
            ds = torch.empty((3,), dtype=torch.float32, device=dev)
            wsb = lsa.dit_quant_fp8_workspace_bytes(n)
            ws = torch.empty((wsb // 4 + 1,), dtype=torch.float32, device=dev)
            for i in range(3):
                lsa.dit_quant_fp8(x[i], codes[i], ds[i:i + 1], n, ws, wsb, stream)
            del x
            call = lambda: lsa.dit_attn_fwd(codes[0], codes[1], codes[2], out, lse, B, H, S, D, w.scale,
                                            lsa.DIT_FP8_E4M3, ds, stream)
        else:
            call = lambda: lsa.dit_attn_fwd(x[0], x[1], x[2], out, lse, B, H, S, D, w.scale, lsa.DIT_BF16, None,
                                            stream)
        ms = _time_calls(call, stream, ranks, reps)
        tf = w.flops * ranks.world / (ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
        res[name + ("_e4m3" if fp8 else "_bf16")] = {
            "B": B, "H": H, "S": S, "D": D, "ms": round(ms, 4), "tflops": round(tf, 2),
            "frac": round(tf / peak, 4),
            "peak": round(peak, 1), "peak_source": f"{src} bf16_tflops (burst)" + (" x 2" if fp8 else "")}
        del out, lse
        if fp8:
            del codes, ds, ws
        else:
            del x
        torch.cuda.empty_cache()
    return res


def run_ring_fused(lsa, step, stream, ranks, reps: int = 10):
    """The same chunked pass with fused ring steps: dit_attn_acc_init + n x
    dit_attn_fwd_chunk_acc into an fp32 accumulator (reported beside the step, not in it)."""
    import torch
    w = step.w
    B, H, S, D = w.B, w.H, w.S, w.D
    acc = torch.empty((B, H, S, D), dtype=torch.float32, device=step.q.device)
    acc_lse = torch.empty((B, H, S), dtype=torch.float32, device=step.q.device)

    def one():
        lsa.dit_attn_acc_init(acc, acc_lse, B, H, S, D, stream)
        for a, b in step.bounds:
            lsa.dit_attn_fwd_chunk_acc(step.q, step.k, step.v, acc, acc_lse, B, H, S, S, D, a, b, w.scale,
                                       lsa.DIT_BF16, None, stream)

    with torch.cuda.stream(stream):
        for _ in range(2):
            one()
        stream.synchronize()
        ranks.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            one()
        t1.record(stream)
    stream.synchronize()
    ms = ranks.max(t0.elapsed_time(t1)) / reps
    return {"ms": round(ms, 4), "tflops": round(w.flops * ranks.world / (ms * 1e-3) / 1e12, 2),
            "calls": "dit_attn_acc_init + %d x dit_attn_fwd_chunk_acc" % len(step.bounds)}


def run_e2e(args, lsa, step, data, stream, dev, ranks):
    import torch
    w = step.w
    host_in = [torch.from_numpy(data[n + "_bits"].view(np.int16)).view(torch.bfloat16).pin_memory() for n in "qkv"]
    host_out = torch.empty(step.out.shape, dtype=torch.bfloat16).pin_memory()
    host_lse = torch.empty(step.lse.shape, dtype=torch.float32).pin_memory()
    outs = [(host_out, step.out), (host_lse, step.lse)]
    if step.bounds:
        host_mout = torch.empty(step.mout.shape, dtype=torch.bfloat16).pin_memory()
        host_mlse = torch.empty(step.mlse.shape, dtype=torch.float32).pin_memory()
        outs += [(host_mout, step.mout), (host_mlse, step.mlse)]
    if step.fp8:
        host_o8 = torch.empty(step.out8.shape, dtype=torch.bfloat16).pin_memory()
        outs += [(host_o8, step.out8)]
    n_steps = max(3, min(args.steps, 10))
    BH = w.B * w.H
    if args.e2e_groups > 0:
        G = max(1, min(args.e2e_groups, BH))
    else:
        # as many whole heads per group as one wave of work units (256 query rows of one
        # head, one per SM) holds: small groups overlap copies best, a partial second wave
        # would leave SMs idle
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        per_group = max(1, sms // ((w.S + 255) // 256))
        G = (BH + per_group - 1) // per_group
    cuts = [min(BH, g * ((BH + G - 1) // G)) for g in range(G + 1)]
    c_in, c_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    fp8_outs = [(h, d) for h, d in outs if step.fp8 and d is step.out8]
    head_outs = [(h, d) for h, d in outs if not (step.fp8 and d is step.out8)]

    def rows(t, g0, g1):
        return t.view(BH, -1)[g0:g1]

    def one():
        # Head groups in a three-stream pipeline: the H2D copy of group g+1 and the D2H copy
        # of group g-1 run on the copy engines while the kernels of group g run.
        start = torch.cuda.Event()
        start.record(stream)
        for st in (c_in, c_out):
            st.wait_event(start)
        for g in range(G):
            g0, g1 = cuts[g], cuts[g + 1]
            if g1 <= g0:
                continue
            cs = stream
            with torch.cuda.stream(c_in):
                for h, d in zip(host_in, (step.q, step.k, step.v)):
                    rows(d, g0, g1).copy_(rows(h, g0, g1), non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(c_in)
            cs.wait_event(arrived)
            step.run_heads(cs, g0, g1)
            done = torch.cuda.Event()
            done.record(cs)
            c_out.wait_event(done)
            with torch.cuda.stream(c_out):
                for h, d in head_outs:
                    rows(h, g0, g1).copy_(rows(d, g0, g1), non_blocking=True)
        if step.fp8:          # per-tensor scales need the whole tensors: after the last group
            step.run_fp8(stream)
            done = torch.cuda.Event()
            done.record(stream)
            c_out.wait_event(done)
            with torch.cuda.stream(c_out):
                for h, d in fp8_outs:
                    h.copy_(d, non_blocking=True)
        end = torch.cuda.Event()
        end.record(c_out)
        stream.wait_event(end)

    with torch.cuda.stream(stream):
        step.run(stream)                       # whole-tensor calls, for the check below
        ref = [d.clone() for _, d in outs]
        one()
        stream.synchronize()
        ranks.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n_steps):
            one()
        t1.record(stream)
    stream.synchronize()
    ms = ranks.max(t0.elapsed_time(t1)) / n_steps
    # the head-group calls must give the whole-tensor calls' results bit for bit
    same = all(torch.equal(h, r.cpu()) for (h, _), r in zip(outs, ref))
    del ref
    bi = sum(h.numel() * h.element_size() for h in host_in)
    bo = sum(h.numel() * h.element_size() for h, _ in outs)
    return {"value": round(step.flops * ranks.world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "steps": n_steps, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "head_groups": G, "pipeline": "H2D / kernels / D2H on three streams, per head group",
            "matches_whole_tensor_calls": bool(same)}


# ----------------------------------------------------------------------------- oracle (CPU)
def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(w, data, rows, heads):
    """Time the fp64 oracle on the given query rows of the given heads (full KV range)."""
    import oracle
    q = data["q"][:, heads]
    k = data["k"][:, heads]
    v = data["v"][:, heads]
    t = time.perf_counter()
    oracle.attention(q, k, v, w.scale, rows=rows)
    dt = time.perf_counter() - t
    flops = 4.0 * w.B * len(heads) * len(rows) * w.S * w.D
    return flops, dt


def cpu_baseline(w, seconds: float):
    """The oracle as it stands, on a bounded sample of the workload sized to ~`seconds`."""
    data = make_qkv(w)
    heads = list(range(w.H))
    rows = list(range(0, min(w.S, 64)))
    flops, dt = oracle_sample(w, data, rows, heads[:1])
    per_row_head = dt / len(rows)
    n_rows = int(max(64, min(w.S, seconds / max(per_row_head * w.H, 1e-9))))
    rows = list(range(n_rows))
    flops, dt = oracle_sample(w, data, rows, heads)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"fp64 oracle, {w.B} batch x {w.H} heads x first {n_rows} query rows x all {w.S} keys "
                      f"of {w.name} ({flops:.3e} FLOP)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    data = make_qkv(w)
    heads = list(range(w.H))
    # size one step to ~ args.ref_step_seconds of CPU work
    _, dt = oracle_sample(w, data, list(range(32)), [0])
    n_rows = int(max(16, min(w.S, args.ref_step_seconds / max(dt / 32 * w.H, 1e-9))))
    rows = list(range(n_rows))
    for _ in range(args.warmup):
        oracle_sample(w, data, rows[:16], heads[:1])
    times, flops = [], 0.0
    for _ in range(args.steps):
        f, dt = oracle_sample(w, data, rows, heads)
        times.append(dt)
        flops = f
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = (f"per step: fp64 oracle on {w.B} batch x {w.H} heads x first {n_rows} query rows x all {w.S} keys "
              f"of {w.name} ({flops:.3e} FLOP)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) rounded to bf16)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "D": w.D, "scale": w.scale},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="flux_2048", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--mode", default="replicas", choices=("replicas",) + SEQPAR_MODES,
                    help="replicas: one independent batch per rank (default); ring / ring_peers / ulysses / "
                         "ulysses_peers: one sequence split across the ranks by that sequence-parallel form")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU work of the oracle baseline sample")
    ap.add_argument("--ref-step-seconds", type=float, default=6.0, help="CPU work per --impl reference step")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-forwards", action="store_true",
                    help="leave out the per-workload forward timings reported beside the step")
    ap.add_argument("--e2e-groups", type=int, default=0,
                    help="head groups of the end-to-end pipeline (copies of one group overlap kernels of another);"
                         " 0 = about one wave of work units per group")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, local_rank, world = rank_info()
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.mode != "replicas":
        run_seqpar(args, rank, local_rank, world)
    else:
        run_ours(args, rank, local_rank, world)


if __name__ == "__main__":
    main()
