"""The Ulysses re-partition across ranks (gloo on CPU, world sizes 1, 2 and 4).

The driver is plumbing: the all-to-all exchanges, the batch/peer transposes and the
segmented layout it hands to the attention.  Here the two device operations are done on the
host by the test (numpy chunk transpose; the fp64 oracle on the segmented layout, unpacked
row by row with the index rule the C entry point documents), so the exchange schedule and
the layout conventions are checked without a GPU: every rank's rows must equal the oracle's
attention over the whole sequence."""

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


class OracleUlyssesOps:
    """Device operations of the driver, on the host (test only)."""

    def __init__(self, scale):
        self.scale = scale
        self.seen = []

    def swap01(self, src, dst, d0, d1, chunk_elems):
        import torch
        a = src.reshape(d0, d1, chunk_elems).numpy()
        dst.copy_(torch.from_numpy(np.ascontiguousarray(a.transpose(1, 0, 2)).reshape(-1)))

    def attention_seg(self, q, k, v, out, lse, B, H, S, D, seg):
        import oracle
        import torch
        self.seen.append((B, H, S, D, seg))
        BH = B * H

        def unseg(x):              # [S/seg][BH][seg][D] -> [BH][S][D], row r at ((r//seg)*BH + bh)*seg + r%seg
            a = x.numpy().reshape(S // seg, BH, seg, D)
            return a.transpose(1, 0, 2, 3).reshape(1, BH, S, D)

        o, l = oracle.attention(unseg(q), unseg(k), unseg(v), self.scale)
        o = o.reshape(BH, S // seg, seg, D).transpose(1, 0, 2, 3).reshape(-1)
        out.copy_(torch.from_numpy(o.astype(np.float32)))
        if lse is not None:
            l = l.reshape(BH, S // seg, seg).transpose(1, 0, 2).reshape(-1)
            lse.copy_(torch.from_numpy(l.astype(np.float32)))


def _full(B, H, S, D, seed=0):
    rng = np.random.default_rng(seed)
    return [rng.normal(size=(B, H, S, D)) for _ in range(3)]


def _worker(rank, world, port, B, H, S_loc, D, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from long_sequence_attention_b200.ulysses import ulysses_attention_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    q, k, v = _full(B, H, world * S_loc, D)
    rows = slice(rank * S_loc, (rank + 1) * S_loc)
    loc = [torch.from_numpy(np.ascontiguousarray(x[:, :, rows]).astype(np.float32)) for x in (q, k, v)]
    ops = OracleUlyssesOps(0.2)
    out, lse = ulysses_attention_dist(*loc, 0.2, ops=ops, out_dtype=torch.float32)
    dist.barrier()
    dist.destroy_process_group()
    assert ops.seen == [(B, H // world, world * S_loc, D, S_loc)]
    np.save(os.path.join(out_dir, f"out{rank}.npy"), out.numpy())
    np.save(os.path.join(out_dir, f"lse{rank}.npy"), lse.numpy())


@pytest.mark.parametrize("world,B,H,S_loc", [(2, 1, 4, 128), (2, 2, 2, 128), (4, 3, 4, 128), (1, 2, 3, 50)])
def test_ulysses_matches_oracle(tmp_path, world, B, H, S_loc):
    import torch.multiprocessing as mp
    import oracle
    D = 8
    mp.spawn(_worker, args=(world, _free_port(), B, H, S_loc, D, str(tmp_path)), nprocs=world, join=True)
    q, k, v = [x.astype(np.float32).astype(np.float64) for x in _full(B, H, world * S_loc, D)]
    ro, rl = oracle.attention(q, k, v, 0.2)
    for r in range(world):
        rows = slice(r * S_loc, (r + 1) * S_loc)
        assert np.allclose(np.load(tmp_path / f"out{r}.npy"), ro[:, :, rows], rtol=0, atol=1e-6)
        assert np.allclose(np.load(tmp_path / f"lse{r}.npy"), rl[:, :, rows], rtol=0, atol=1e-5)


def _bad_worker(rank, world, port, H, S_loc, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from long_sequence_attention_b200.ulysses import ulysses_attention_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    x = torch.zeros(1, H, S_loc, 8)
    msg = ""
    try:
        ulysses_attention_dist(x, x, x, 0.2, ops=OracleUlyssesOps(0.2))
    except ValueError as e:
        msg = str(e)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"err{rank}.txt"), "w") as f:
        f.write(msg)


@pytest.mark.parametrize("H,S_loc,word", [(3, 128, "divide"), (4, 100, "multiple of 128")])
def test_ulysses_rejects_bad_shapes(tmp_path, H, S_loc, word):
    import torch.multiprocessing as mp
    mp.spawn(_bad_worker, args=(2, _free_port(), H, S_loc, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert word in open(tmp_path / f"err{r}.txt").read()


# ------------------------------------------------------------------ peer-memory Ulysses step
class SharedMemoryPeerOps:
    """Peer memory emulated with CPU tensors in shared memory (test only): every process maps
    every rank's buffers; an exported "handle" names a buffer, importing it gives this
    process's address of that buffer, and the launch computes its head group with the fp64
    oracle, reading the parts through the addresses it is given and writing each output row
    into the part it belongs to, as the fused kernel does."""

    def __init__(self, rank, buffers, scale):
        self.rank, self.scale = rank, scale
        self.by_name = {}
        self.by_ptr = {}
        for r, bufs in enumerate(buffers):
            for i, t in enumerate(bufs):
                self.by_name[(r, i)] = t
                self.by_ptr[t.data_ptr()] = t
        self.launches = []

    def export(self, t):
        for (r, i), u in self.by_name.items():
            if u.data_ptr() == t.data_ptr():
                return f"{r}:{i}".encode().ljust(64, b"\0"), 0
        raise AssertionError("export of an unknown buffer")

    def import_(self, rank, handle, offset):
        r, i = (int(x) for x in handle.rstrip(b"\0").decode().split(":"))
        assert r == rank, "a handle opened as another rank's"
        return self.by_name[(r, i)].data_ptr() + offset

    def sync(self):
        pass

    def launch(self, qs, ks, vs, outs, lses, B, H, h0, Hp, rows, D, scale):
        import oracle
        import torch
        self.launches.append((h0, Hp))
        T = lambda p: self.by_ptr[p]
        heads = slice(h0, h0 + Hp)
        q = torch.cat([T(p)[:, heads] for p in qs], dim=2).numpy()
        k = torch.cat([T(p)[:, heads] for p in ks], dim=2).numpy()
        v = torch.cat([T(p)[:, heads] for p in vs], dim=2).numpy()
        o, l = oracle.attention(q, k, v, scale)
        for part, (po, pl) in enumerate(zip(outs, lses)):
            sl = slice(part * rows, (part + 1) * rows)
            T(po)[:, heads] = torch.from_numpy(o[:, :, sl].astype(np.float32))
            T(pl)[:, heads] = torch.from_numpy(l[:, :, sl].astype(np.float32))


def _peers_worker(rank, world, port, buffers, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from long_sequence_attention_b200.ulysses import ulysses_attention_peers
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ops = SharedMemoryPeerOps(rank, buffers, 0.2)
    q, k, v, out, lse = buffers[rank]
    ulysses_attention_peers(q, k, v, 0.2, ops=ops, out=out, lse=lse)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"launch{rank}.txt"), "w") as f:
        f.write(repr(ops.launches))


@pytest.mark.parametrize("world,B,H,S_loc", [(2, 1, 4, 128), (4, 2, 4, 128), (3, 1, 6, 256)])
def test_peer_ulysses_schedule_matches_oracle(tmp_path, world, B, H, S_loc):
    """Every rank's output rows come from every rank's launch; after the driver returns they
    must all be there (the second barrier) and equal the oracle over the whole sequence."""
    import torch
    import torch.multiprocessing as mp
    import oracle
    D = 8
    q, k, v = [x.astype(np.float32) for x in _full(B, H, world * S_loc, D)]
    buffers = []
    for r in range(world):
        rows = slice(r * S_loc, (r + 1) * S_loc)
        bufs = [torch.from_numpy(np.ascontiguousarray(x[:, :, rows])).share_memory_() for x in (q, k, v)]
        bufs.append(torch.full((B, H, S_loc, D), float("nan")).share_memory_())
        bufs.append(torch.full((B, H, S_loc), float("nan")).share_memory_())
        buffers.append(bufs)
    mp.spawn(_peers_worker, args=(world, _free_port(), buffers, str(tmp_path)), nprocs=world, join=True)
    ro, rl = oracle.attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), 0.2)
    Hp = H // world
    for r in range(world):
        rows = slice(r * S_loc, (r + 1) * S_loc)
        assert np.allclose(buffers[r][3].numpy(), ro[:, :, rows], rtol=0, atol=1e-6)
        assert np.allclose(buffers[r][4].numpy(), rl[:, :, rows], rtol=0, atol=1e-5)
        assert open(tmp_path / f"launch{r}.txt").read() == repr([(r * Hp, Hp)])
