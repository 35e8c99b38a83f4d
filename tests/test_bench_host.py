"""Host logic of bench.py that needs no GPU: the multi-rank plumbing (gloo, world size 2),
replica seeding, and the reference arm (the fp64 oracle timed on the host cores), both as a
single process and under torchrun with two ranks."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ranks_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks(world, backend="gloo", timeout_s=60)
    r.init()
    r.barrier()
    got = r.max(10.0 + 3.0 * rank)          # rank-dependent "elapsed time"
    seed = bench.replica_seed_offset(rank)
    r.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": got, "seed": seed}, f)


def test_ranks_max_over_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_ranks_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [x["max"] for x in res] == [13.0, 13.0]           # every rank sees the max over ranks
    assert res[0]["seed"] != res[1]["seed"]                   # replicas draw different batches


def test_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks(1)
    r.init()
    r.barrier()
    assert r.max(4.5) == 4.5
    r.close()


def _json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_reference_arm_single_process():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
           "--warmup", "3", "--ref-step-seconds", "0.2"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr
    lines = _json_lines(out.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "tiny"


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
           "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
           "--ref-step-seconds", "0.2"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr
    lines = _json_lines(out.stdout)
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2      # rank 0 alone prints


def test_seqpar_blocks_and_launch_counts():
    sys.path.insert(0, ROOT)
    import bench
    # the NCCL ring takes any split; the last rank gets the remainder
    blocks, why = bench.seqpar_blocks("ring", 1000, 24, 3)
    assert why is None and blocks == [(0, 333), (333, 666), (666, 1000)]
    # FLUX-2048 over 4 ranks: 4224 rows each (33 tiles); over 8 ranks 2112 is not a tile multiple
    blocks, why = bench.seqpar_blocks("ulysses", 16896, 24, 4)
    assert why is None and blocks[1] == (4224, 8448)
    for mode in ("ulysses", "ulysses_peers", "ring_peers"):
        assert bench.seqpar_blocks(mode, 16896, 24, 8)[1] is not None
        assert bench.seqpar_blocks(mode, 16896, 24, 1)[0] == [(0, 16896)]
    assert bench.seqpar_blocks("ulysses", 4096, 24, 16)[1] is not None          # 16 does not divide 24
    assert bench.seqpar_blocks("ulysses_peers", 16384, 32, 16)[1] is not None    # more than 8 ranks
    assert bench.seqpar_launches("ring", 1, 4) == 6
    assert bench.seqpar_launches("ulysses", 2, 4) == 6 and bench.seqpar_launches("ulysses", 1, 4) == 1


def test_seqpar_mode_reports_an_unsupported_split():
    """Under torchrun with two ranks, a split the mode cannot take (S/P not a multiple of 128)
    prints one 'unavailable' line from rank 0 and exits 0 on every rank before any GPU work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
           "--mode", "ulysses", "--workload", "sd3_1024", "--steps", "3", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr
    lines = _json_lines(out.stdout)
    assert len(lines) == 1 and "unavailable" in lines[0] and lines[0]["n_gpus"] == 2
