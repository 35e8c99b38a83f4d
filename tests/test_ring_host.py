"""The KV ring's send/recv schedule across ranks (gloo on CPU, world sizes 2-4).

The ring driver is plumbing: buffers, the order of sends and receives, block lengths.  Here
its step functions are the fp64 oracle (attention over one block, then the exact LSE merge
into the accumulator), passed in by the test, so the schedule is checked without a GPU: the
result on every rank must equal the oracle's attention over the concatenation of all
ranks' blocks.  A block sent to the wrong rank, received twice, or read after it was
overwritten changes that result."""

import json
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleRingOps:
    """Ring step functions on the fp64 oracle (test only)."""

    def __init__(self, scale, k_blocks):
        self.scale = scale
        self.k_blocks = k_blocks
        self.owners_seen = []

    def init(self, acc, lse):
        acc.zero_()
        lse.fill_(-np.inf)

    def step(self, q, k_blk, v_blk, s_kv, acc, lse, descale):
        import oracle
        import torch
        kb = k_blk.numpy()
        self.owners_seen.append(next((r for r, blk in enumerate(self.k_blocks)
                                      if blk.shape == kb.shape and np.array_equal(blk, kb)), -1) if s_kv else None)
        if s_kv == 0:
            return
        o, l = oracle.attention(q.numpy(), k_blk.numpy(), v_blk.numpy(), self.scale)
        mo, ml = oracle.merge([acc.numpy().astype(np.float64), o], [lse.numpy().astype(np.float64), l])
        acc.copy_(torch.from_numpy(mo))
        lse.copy_(torch.from_numpy(ml))

    def finish(self, acc, lse):
        return acc, lse


def _blocks(lens, B=1, H=2, D=8, seed=0):
    """Q, K, V over all ranks' rows and the row offsets of each rank's block."""
    rng = np.random.default_rng(seed)
    S = sum(lens)
    q = rng.normal(size=(B, H, S, D))
    k = rng.normal(size=(B, H, S, D))
    v = rng.normal(size=(B, H, S, D))
    offs = np.cumsum([0] + list(lens))
    return q, k, v, offs


def _ring_worker(rank, world, port, lens, out_dir, pass_lens):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from long_sequence_attention_b200.ring import ring_attention_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    q, k, v, offs = _blocks(lens)
    a, b = offs[rank], offs[rank + 1]
    scale = 0.3
    ops = OracleRingOps(scale, [k[:, :, offs[i]:offs[i + 1]] for i in range(world)])
    # this rank's queries are its own rows; its K/V block the same rows
    qt = torch.from_numpy(np.ascontiguousarray(q[:, :, a:b]))
    kt = torch.from_numpy(np.ascontiguousarray(k[:, :, a:b]))
    vt = torch.from_numpy(np.ascontiguousarray(v[:, :, a:b]))
    out, lse = ring_attention_dist(qt, kt, vt, scale, ops=ops, block_lens=list(lens) if pass_lens else None)
    dist.barrier()
    dist.destroy_process_group()
    np.save(os.path.join(out_dir, f"out{rank}.npy"), out.numpy())
    np.save(os.path.join(out_dir, f"lse{rank}.npy"), lse.numpy())
    with open(os.path.join(out_dir, f"owners{rank}.json"), "w") as f:
        json.dump(ops.owners_seen, f)


@pytest.mark.parametrize("lens,pass_lens", [
    ((64, 64), False),
    ((37, 50, 41), False),                  # S not divisible by P: uneven blocks
    ((16, 0, 23, 9), True),                 # an empty block travels too (skipped by both ends)
])
def test_ring_schedule_matches_oracle(tmp_path, lens, pass_lens):
    import torch.multiprocessing as mp
    import oracle
    world = len(lens)
    mp.spawn(_ring_worker, args=(world, _free_port(), lens, str(tmp_path), pass_lens), nprocs=world, join=True)
    q, k, v, offs = _blocks(lens)
    ref_o, ref_l = oracle.attention(q, k, v, 0.3)
    for r in range(world):
        a, b = offs[r], offs[r + 1]
        o = np.load(tmp_path / f"out{r}.npy")
        l = np.load(tmp_path / f"lse{r}.npy")
        assert np.allclose(o, ref_o[:, :, a:b], rtol=0, atol=1e-6)
        assert np.allclose(l, ref_l[:, :, a:b], rtol=0, atol=1e-5)
        owners = json.load(open(tmp_path / f"owners{r}.json"))
        # step t works on the block of rank (r - t) mod P
        want = [(r - t) % world if lens[(r - t) % world] else None for t in range(world)]
        assert owners == want, (r, owners, want)


def test_ring_single_rank_is_one_step(tmp_path):
    import torch.multiprocessing as mp
    import oracle
    lens = (40,)
    mp.spawn(_ring_worker, args=(1, _free_port(), lens, str(tmp_path), False), nprocs=1, join=True)
    q, k, v, _ = _blocks(lens)
    ref_o, ref_l = oracle.attention(q, k, v, 0.3)
    assert np.allclose(np.load(tmp_path / "out0.npy"), ref_o, rtol=0, atol=1e-6)
    assert json.load(open(tmp_path / "owners0.json")) == [0]


def _ring_peers_worker(rank, world, port, buffers, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    from long_sequence_attention_b200.ring import ring_attention_peers
    from test_ulysses_host import SharedMemoryPeerOps
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ops = SharedMemoryPeerOps(rank, buffers, 0.3)
    q, k, v, out, lse = buffers[rank]
    ring_attention_peers(q, k, v, 0.3, ops=ops, out=out, lse=lse)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"launch{rank}.txt"), "w") as f:
        f.write(repr(ops.launches))


@pytest.mark.parametrize("world,S_loc", [(2, 128), (3, 256)])
def test_ring_peers_matches_oracle(tmp_path, world, S_loc):
    """The ring without a ring: each rank's launch reads every rank's K/V block in place (here
    shared CPU memory stands in for peer memory) and writes only its own rows."""
    import torch
    import torch.multiprocessing as mp
    import oracle
    B, H, D = 1, 2, 8
    q, k, v, offs = _blocks([S_loc] * world, B=B, H=H, D=D)
    buffers = []
    for r in range(world):
        rows = slice(offs[r], offs[r + 1])
        bufs = [torch.from_numpy(np.ascontiguousarray(x[:, :, rows]).astype(np.float32)).share_memory_()
                for x in (q, k, v)]
        bufs.append(torch.full((B, H, S_loc, D), float("nan")).share_memory_())
        bufs.append(torch.full((B, H, S_loc), float("nan")).share_memory_())
        buffers.append(bufs)
    mp.spawn(_ring_peers_worker, args=(world, _free_port(), buffers, str(tmp_path)), nprocs=world, join=True)
    f32 = lambda x: x.astype(np.float32).astype(np.float64)
    ro, rl = oracle.attention(f32(q), f32(k), f32(v), 0.3)
    for r in range(world):
        rows = slice(offs[r], offs[r + 1])
        assert np.allclose(buffers[r][3].numpy(), ro[:, :, rows], rtol=0, atol=1e-6)
        assert np.allclose(buffers[r][4].numpy(), rl[:, :, rows], rtol=0, atol=1e-5)
        assert open(tmp_path / f"launch{r}.txt").read() == repr([(0, H)])
