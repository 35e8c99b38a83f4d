"""C-ABI checks that need no GPU: the library loads, exports every declared symbol, and
host-side validation rejects bad arguments before anything reaches CUDA."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dit_attn.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dit_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    import long_sequence_attention_b200 as lsa
    return lsa


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("dit_attn_fwd", "dit_attn_fwd_chunk", "dit_attn_merge", "dit_quant_fp8",
              "dit_quant_fp8_workspace_bytes", "dit_device_status", "dit_status_str", "dit_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in _declared():
        assert hasattr(raw, name), name


def test_only_dit_symbols_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True, text=True).stdout
    syms = [l.split()[-1] for l in out.splitlines() if l.strip()]
    assert syms and all(s.startswith("dit_") for s in syms), syms


def test_status_strings_and_version(lib):
    assert lib.status_str(0) == "DIT_OK"
    assert lib.status_str(5) == "DIT_ERR_TIMEOUT"
    assert lib.status_str(5 | (3 << 8)) == "DIT_ERR_TIMEOUT"
    assert lib.dit_version() >= 100


# Fake, 256-byte aligned, non-null "device" addresses: validation must reject the call
# before touching them.  Every call below has at least one invalid argument, so nothing is
# ever launched on these addresses (not even on a machine with a GPU).
A = 1 << 40
Bp = A + (1 << 30)
Cp = A + (2 << 30)
O = A + (3 << 30)
L = A + (4 << 30)


def _chunk(lib, **kw):
    args = dict(q=A, k=Bp, v=Cp, out=O, lse=L, B=1, H=2, S_q=256, S_kv=256, D=64, k0=0, k1=256,
                scale=0.125, dtype=0, out_dtype=2, descale=None, stream=None)
    args.update(kw)
    return lib.lib.dit_attn_fwd_chunk(args["q"], args["k"], args["v"], args["out"], args["lse"], args["B"],
                                      args["H"], args["S_q"], args["S_kv"], args["D"], args["k0"], args["k1"],
                                      args["scale"], args["dtype"], args["out_dtype"], args["descale"],
                                      args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(B=0), 1), (dict(H=0), 1), (dict(S_q=0), 1),
    (dict(S_kv=0), 1), (dict(k0=-1), 1), (dict(k0=10, k1=5), 1), (dict(k1=257), 1),
    (dict(scale=0.0), 1), (dict(scale=-1.0), 1), (dict(scale=float("inf")), 1), (dict(scale=float("nan")), 1),
    (dict(dtype=7), 1), (dict(out_dtype=1), 1), (dict(D=96), 2), (dict(D=256), 2),
    (dict(dtype=1, D=64, descale=A + 64), 2), (dict(dtype=1, D=128, descale=None), 1),
    (dict(q=A + 8), 3), (dict(out=O + 4), 3), (dict(lse=L + 2), 3),
    (dict(out=A + 128), 1),            # output overlaps q
    (dict(lse=O + 64), 1),             # lse overlaps out
])
def test_chunk_validation(lib, kw, code):
    assert _chunk(lib, **kw) == code


def test_fwd_validation(lib):
    f = lib.lib.dit_attn_fwd
    assert f(None, Bp, Cp, O, L, 1, 2, 256, 64, 0.125, 0, None, None) == 1
    assert f(A, Bp, Cp, O, L, 1, 2, 256, 80, 0.125, 0, None, None) == 2


def test_merge_validation(lib):
    vp = ctypes.c_void_p
    outs = (vp * 2)(Bp, Cp)
    lses = (vp * 2)(L, L + 4096)
    m = lib.lib.dit_attn_merge
    assert m(outs, lses, 0, O, None, 1, 2, 8, 64, 2, 0, None) == 1          # n_chunks
    assert m(outs, lses, 17, O, None, 1, 2, 8, 64, 2, 0, None) == 1
    assert m(outs, lses, 2, O, None, 1, 2, 8, 96, 2, 0, None) == 2          # D
    assert m(outs, lses, 2, O, None, 1, 2, 8, 64, 1, 0, None) == 1          # in dtype
    assert m(outs, lses, 2, O + 8, None, 1, 2, 8, 64, 2, 0, None) == 3      # misaligned out
    bad = (vp * 2)(Bp + 4, Cp)
    assert m(bad, lses, 2, O, None, 1, 2, 8, 64, 2, 0, None) == 3
    alias = (vp * 2)(O, Cp)
    assert m(alias, lses, 2, O, None, 1, 2, 8, 64, 2, 0, None) == 1         # out aliases a partial
    null = (vp * 2)(Bp, None)
    assert m(null, lses, 2, O, None, 1, 2, 8, 64, 2, 0, None) == 1


def test_quant_validation(lib):
    q = lib.lib.dit_quant_fp8
    ws = lib.dit_quant_fp8_workspace_bytes(1 << 20)
    assert ws == 4 * 128
    assert lib.dit_quant_fp8_workspace_bytes(1) == 4
    assert lib.dit_quant_fp8_workspace_bytes(1 << 40) == 4 * 1184
    assert q(None, Bp, L, 1 << 20, Cp, ws, None) == 1
    assert q(A, Bp, L, 0, Cp, ws, None) == 1
    assert q(A, Bp, L, 1 << 20, Cp, ws - 4, None) == 1                       # workspace too small
    assert q(A + 2, Bp, L, 1 << 20, Cp, ws, None) == 3
    assert q(A, A + 64, L, 1 << 20, Cp, ws, None) == 1                       # output overlaps input


def test_selftest_validation(lib):
    assert lib.lib.dit_selftest_wait_timeout(0, None) == 1
    assert lib.lib.dit_selftest_wait_timeout(10 ** 9, None) == 1


def test_sm_reserve_validation(lib):
    assert lib.lib.dit_set_sm_reserve(-1) == 1
    assert lib.lib.dit_set_sm_reserve(1025) == 1
    assert lib.lib.dit_set_sm_reserve(8) == 0
    assert lib.lib.dit_set_sm_reserve(0) == 0


# Every call below also carries at least one invalid argument (see the note above).
def test_block_fp8_validation(lib):
    qb = lib.lib.dit_quant_fp8_blocks
    assert qb(None, Bp, L, 1, 2, 256, 128, None) == 1
    assert qb(A, Bp, L, 1, 2, 256, 4, None) == 1                             # D < 8
    assert qb(A, Bp, L, 1, 2, 256, 12, None) == 2                            # D % 8
    assert qb(A, Bp, L, 1, 2, 256, 136, None) == 2                           # D > 128
    assert qb(A + 2, Bp, L, 1, 2, 256, 128, None) == 3
    assert qb(A, A + 64, L, 1, 2, 256, 128, None) == 1                       # codes overlap input
    fb = lib.lib.dit_attn_fwd_fp8_blocks
    assert fb(A, Bp, Cp, L, None, L + 4096, O, None, 1, 2, 256, 256, 128, 0, 256, 0.1, 0, None) == 1
    assert fb(A, Bp, Cp, L, L + 1024, L + 4096, O, None, 1, 2, 256, 256, 128, 64, 256, 0.1, 0, None) == 2
    assert fb(A, Bp, Cp, L, L + 1024, L + 4096, O, None, 1, 2, 256, 256, 64, 0, 256, 0.1, 0, None) == 2


def test_seg_and_swap_validation(lib):
    sg = lib.lib.dit_attn_fwd_seg
    assert sg(A, Bp, Cp, O, L, 1, 2, 512, 128, 0, 0.1, 0, 0, None, None) == 1        # seg < 1
    assert sg(A, Bp, Cp, O, L, 1, 2, 512, 128, 300, 0.1, 0, 0, None, None) == 1      # S % seg
    assert sg(A, Bp, Cp, O, L, 1, 2, 512, 128, 64, 0.1, 0, 0, None, None) == 2       # seg % 128
    sw = lib.lib.dit_swap01_chunks
    assert sw(None, Bp, 2, 2, 64, None) == 1
    assert sw(A, Bp, 2, 2, 8, None) == 1                                     # chunk < 16 bytes
    assert sw(A, Bp, 2, 2, 24, None) == 2                                    # chunk % 16
    assert sw(A + 8, Bp, 2, 2, 64, None) == 3
    assert sw(A, A + 64, 2, 2, 64, None) == 1                                # dst overlaps src


def test_na3d_validation(lib):
    na = lib.lib.dit_na3d_fwd
    assert na(None, Bp, Cp, O, L, 1, 2, 3, 4, 5, 64, 3, 3, 3, 0.1, None) == 1
    assert na(A, Bp, Cp, O, L, 1, 2, 3, 4, 5, 64, 2, 3, 3, 0.1, None) == 1   # even window
    assert na(A, Bp, Cp, O, L, 1, 2, 3, 4, 5, 64, 3, 5, 3, 0.1, None) == 1   # window > grid
    assert na(A, Bp, Cp, O, L, 1, 2, 3, 4, 5, 96, 3, 3, 3, 0.1, None) == 2   # D
    assert na(A + 8, Bp, Cp, O, L, 1, 2, 3, 4, 5, 64, 3, 3, 3, 0.1, None) == 3
    assert na(A, Bp, Cp, O, L, 1, 2, 3, 4, 5, 64, 3, 3, 3, 0.0, None) == 1   # scale
    assert na(A, Bp, Cp, O, L, 1, 2, 3, 4, 5, 64, 3, 3, 3, 1e-21, None) == 1  # scale below the penalty's range


def test_parts_validation(lib):
    vp = ctypes.c_void_p
    arr = lambda *xs: (vp * len(xs))(*xs)
    pf = lib.lib.dit_attn_fwd_parts
    q2, k2, v2, o2 = arr(A, A + (1 << 28)), arr(Bp, Bp + (1 << 28)), arr(Cp, Cp + (1 << 28)), arr(O, O + (1 << 28))
    assert pf(q2, 0, k2, v2, 2, o2, None, 1, 4, 0, 2, 256, 128, 0.1, None) == 1          # no query blocks
    assert pf(q2, 2, k2, v2, 9, o2, None, 1, 4, 0, 2, 256, 128, 0.1, None) == 1          # too many blocks
    assert pf(q2, 2, k2, v2, 2, o2, None, 1, 4, 0, 2, 192, 128, 0.1, None) == 2          # 192 rows per block
    assert pf(q2, 2, k2, v2, 2, o2, None, 1, 4, 3, 2, 256, 128, 0.1, None) == 1          # heads past part_H
    assert pf(arr(A, None), 2, k2, v2, 2, o2, None, 1, 4, 0, 2, 256, 128, 0.1, None) == 1
    assert pf(arr(A + 8, A + (1 << 28)), 2, k2, v2, 2, o2, None, 1, 4, 0, 2, 256, 128, 0.1, None) == 3
    assert pf(q2, 2, k2, v2, 2, arr(O, A), None, 1, 4, 0, 2, 256, 128, 0.1, None) == 1   # out overlaps q
    fp = ctypes.c_void_p
    larr = lambda *xs: (fp * len(xs))(*xs)
    assert pf(q2, 2, k2, v2, 2, o2, larr(L, A), 1, 4, 0, 2, 256, 128, 0.1, None) == 1          # lse overlaps q
    assert pf(q2, 2, k2, v2, 2, o2, larr(L, Bp + 64), 1, 4, 0, 2, 256, 128, 0.1, None) == 1    # lse overlaps k
    assert pf(q2, 2, k2, v2, 2, o2, larr(L, Cp), 1, 4, 0, 2, 256, 128, 0.1, None) == 1         # lse overlaps v
    assert pf(q2, 2, k2, v2, 2, o2, larr(L, O + 256), 1, 4, 0, 2, 256, 128, 0.1, None) == 1    # lse overlaps out
    assert pf(q2, 2, k2, v2, 2, o2, larr(L, L + 64), 1, 4, 0, 2, 256, 128, 0.1, None) == 1     # lse blocks overlap


def test_acc_and_ipc_validation(lib):
    acc = lib.lib.dit_attn_fwd_chunk_acc
    assert acc(A, Bp, Cp, None, L, 1, 2, 256, 256, 64, 0, 256, 0.125, 0, None, None) == 1
    init = lib.lib.dit_attn_acc_init
    assert init(O, L, 1, 2, 256, 96, None) == 2
    assert init(O + 4, L, 1, 2, 256, 64, None) == 3
    off = ctypes.c_longlong(0)
    assert lib.lib.dit_ipc_export(None, ctypes.create_string_buffer(64), ctypes.byref(off)) == 1
    p, b = ctypes.c_void_p(), ctypes.c_void_p()
    assert lib.lib.dit_ipc_import(None, 0, ctypes.byref(p), ctypes.byref(b)) == 1
    assert lib.lib.dit_ipc_import(ctypes.create_string_buffer(64), -1, ctypes.byref(p), ctypes.byref(b)) == 1
    assert lib.lib.dit_ipc_close(None) == 1
