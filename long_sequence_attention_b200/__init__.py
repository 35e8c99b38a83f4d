"""Python binding of the DiT joint-attention library for B200 (sm_100a).

Argument marshalling only: every computation runs in the CUDA kernels of
``libdit_attn.so`` (built in-tree by ``long_sequence_attention_b200/build.py``).  The C
functions keep their names here (``dit_attn_fwd``, ``dit_attn_fwd_chunk``,
``dit_attn_merge``, ``dit_quant_fp8`` ...); tensors may be passed as torch CUDA tensors or
as raw device addresses (ints).  A non-zero status raises ``DitError``.

Importing this package fails loudly (ImportError) when the library has not been built:
there is no fallback implementation.

The few ``attention`` / ``attention_chunk`` / ``merge`` / ``quantize_fp8`` helpers below
only allocate outputs with torch and call the C entry points.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdit_attn.so")

DIT_BF16, DIT_FP8_E4M3, DIT_FP32 = 0, 1, 2
DIT_OK, DIT_ERR_INVALID_ARG, DIT_ERR_UNSUPPORTED, DIT_ERR_MISALIGNED, DIT_ERR_CUDA, DIT_ERR_TIMEOUT = range(6)


class DitError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {status_str(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python long_sequence_attention_b200/build.py` "
                          "(nvcc, sm_100a). There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
    sz, ull = ctypes.c_size_t, ctypes.c_ulonglong
    lib.dit_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp]
    lib.dit_attn_fwd_chunk.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, vp, vp]
    lib.dit_attn_merge.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i, vp, vp, i, i, i, i, i, i, vp]
    lib.dit_attn_fwd_chunk_acc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, vp]
    lib.dit_attn_acc_init.argtypes = [vp, vp, i, i, i, i, vp]
    lib.dit_quant_fp8_workspace_bytes.argtypes = [ll]
    lib.dit_quant_fp8_workspace_bytes.restype = sz
    lib.dit_quant_fp8.argtypes = [vp, vp, vp, ll, vp, sz, vp]
    lib.dit_quant_fp8_noalloc.argtypes = [vp, vp, vp, ll, vp]
    lib.dit_quant_fp8_noalloc.restype = ctypes.c_int
    lib.dit_device_status.argtypes = [ctypes.POINTER(i), i]
    lib.dit_set_wait_timeout_us.argtypes = [ull]
    lib.dit_selftest_wait_timeout.argtypes = [ull, vp]
    lib.dit_set_sm_reserve.argtypes = [i]
    lib.dit_quant_fp8_blocks.argtypes = [vp, vp, vp, i, i, i, i, vp]
    lib.dit_attn_fwd_seg.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, vp]
    lib.dit_swap01_chunks.argtypes = [vp, vp, ll, ll, ll, vp]
    lib.dit_na3d_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, vp]
    lib.dit_na3d_plan.argtypes = [i, i, i, i, i, i, ctypes.POINTER(i), ctypes.POINTER(ll), ctypes.POINTER(ll)]
    lib.dit_attn_fwd_parts.argtypes = [ctypes.POINTER(vp), i, ctypes.POINTER(vp), ctypes.POINTER(vp), i,
                                       ctypes.POINTER(vp), ctypes.POINTER(vp), i, i, i, i, i, i, f, vp]
    lib.dit_ipc_export.argtypes = [vp, vp, ctypes.POINTER(ll)]
    lib.dit_ipc_import.argtypes = [vp, ll, ctypes.POINTER(vp), ctypes.POINTER(vp)]
    lib.dit_ipc_close.argtypes = [vp]
    lib.dit_attn_fwd_fp8_blocks.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp]
    lib.dit_status_str.argtypes = [i]
    lib.dit_status_str.restype = ctypes.c_char_p
    lib.dit_version.argtypes = []
    for name in ("dit_attn_fwd", "dit_attn_fwd_chunk", "dit_attn_fwd_chunk_acc", "dit_attn_acc_init",
                 "dit_attn_merge", "dit_quant_fp8", "dit_device_status",
                 "dit_set_wait_timeout_us", "dit_selftest_wait_timeout", "dit_version"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load()


def status_str(status: int) -> str:
    return lib.dit_status_str(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != DIT_OK:
        raise DitError(rc, where)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --------------------------------------------------------------------------- C entry points

def dit_attn_fwd(q, k, v, out, lse, B: int, H: int, S: int, D: int, scale: float,
                 dtype: int = DIT_BF16, descale_qkv=None, stream=None) -> None:
    _check(lib.dit_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D, float(scale),
                            dtype, _ptr(descale_qkv), _stream(stream)), "dit_attn_fwd")


def dit_attn_fwd_chunk(q, k, v, out, lse, B: int, H: int, S_q: int, S_kv: int, D: int, k0: int, k1: int,
                       scale: float, dtype: int = DIT_BF16, out_dtype: int = DIT_FP32, descale_qkv=None,
                       stream=None) -> None:
    _check(lib.dit_attn_fwd_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S_q, S_kv, D, k0, k1,
                                  float(scale), dtype, out_dtype, _ptr(descale_qkv), _stream(stream)),
           "dit_attn_fwd_chunk")


def dit_attn_fwd_chunk_acc(q, k, v, acc_out, acc_lse, B: int, H: int, S_q: int, S_kv: int, D: int, k0: int,
                           k1: int, scale: float, dtype: int = DIT_BF16, descale_qkv=None, stream=None) -> None:
    _check(lib.dit_attn_fwd_chunk_acc(_ptr(q), _ptr(k), _ptr(v), _ptr(acc_out), _ptr(acc_lse), B, H, S_q, S_kv, D,
                                      k0, k1, float(scale), dtype, _ptr(descale_qkv), _stream(stream)),
           "dit_attn_fwd_chunk_acc")


def dit_attn_acc_init(acc_out, acc_lse, B: int, H: int, S: int, D: int, stream=None) -> None:
    _check(lib.dit_attn_acc_init(_ptr(acc_out), _ptr(acc_lse), B, H, S, D, _stream(stream)), "dit_attn_acc_init")


def dit_attn_merge(outs: Sequence, lses: Sequence, out, lse, B: int, H: int, S: int, D: int,
                   in_dtype: int = DIT_FP32, out_dtype: int = DIT_BF16, stream=None) -> None:
    n = len(outs)
    arr_o = (ctypes.c_void_p * n)(*[_ptr(o) for o in outs])
    arr_l = (ctypes.c_void_p * n)(*[_ptr(x) for x in lses])
    _check(lib.dit_attn_merge(arr_o, arr_l, n, _ptr(out), _ptr(lse), B, H, S, D, in_dtype, out_dtype,
                              _stream(stream)), "dit_attn_merge")


def dit_quant_fp8_workspace_bytes(n: int) -> int:
    return int(lib.dit_quant_fp8_workspace_bytes(int(n)))


def dit_quant_fp8(x_bf16, x_fp8, descale, n: int, workspace, workspace_bytes: int, stream=None) -> None:
    _check(lib.dit_quant_fp8(_ptr(x_bf16), _ptr(x_fp8), _ptr(descale), int(n), _ptr(workspace),
                             int(workspace_bytes), _stream(stream)), "dit_quant_fp8")


def dit_attn_fwd_seg(q, k, v, out, lse, B: int, H: int, S: int, D: int, seg: int, scale: float,
                     dtype: int = 0, out_dtype: int = 0, descale_qkv=None, stream=None) -> None:
    _check(lib.dit_attn_fwd_seg(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D, seg, float(scale),
                                dtype, out_dtype, _ptr(descale_qkv), _stream(stream)), "dit_attn_fwd_seg")


def dit_attn_fwd_parts(q_parts: Sequence, k_parts: Sequence, v_parts: Sequence, out_parts: Sequence,
                       lse_parts: Optional[Sequence], B: int, part_H: int, h0: int, H: int, part_rows: int, D: int,
                       scale: float, stream=None) -> None:
    """Query blocks q_parts (outputs out_parts, lse_parts) and key blocks k_parts / v_parts;
    the counts are the lengths of the lists."""
    def arr(xs):
        return (ctypes.c_void_p * len(xs))(*[_ptr(x) for x in xs])
    lse_arr = None if lse_parts is None else ctypes.cast(arr(lse_parts), ctypes.POINTER(ctypes.c_void_p))
    _check(lib.dit_attn_fwd_parts(arr(q_parts), len(q_parts), arr(k_parts), arr(v_parts), len(k_parts),
                                  arr(out_parts), lse_arr, B, part_H, h0, H, part_rows, D, float(scale),
                                  _stream(stream)), "dit_attn_fwd_parts")


def dit_ipc_export(ptr) -> Tuple[bytes, int]:
    """(64-byte CUDA IPC handle of the allocation holding ptr, byte offset of ptr in it)."""
    h = ctypes.create_string_buffer(64)
    off = ctypes.c_longlong(0)
    _check(lib.dit_ipc_export(_ptr(ptr), h, ctypes.byref(off)), "dit_ipc_export")
    return h.raw, off.value


def dit_ipc_import(handle: bytes, offset: int) -> Tuple[int, int]:
    """(device address, mapped allocation base) of a buffer exported by another process."""
    p, b = ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib.dit_ipc_import(ctypes.create_string_buffer(handle, 64), int(offset), ctypes.byref(p), ctypes.byref(b)),
           "dit_ipc_import")
    return p.value, b.value


def dit_ipc_close(base: int) -> None:
    _check(lib.dit_ipc_close(base), "dit_ipc_close")


def dit_na3d_fwd(q, k, v, out, lse, B: int, H: int, T: int, Y: int, X: int, D: int, Kt: int, Ky: int, Kx: int,
                 scale: float, stream=None) -> None:
    _check(lib.dit_na3d_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, T, Y, X, D, Kt, Ky, Kx,
                            float(scale), _stream(stream)), "dit_na3d_fwd")


def dit_na3d_plan(T: int, Y: int, X: int, Kt: int, Ky: int, Kx: int):
    """The neighborhood kernel's tiling for a grid and window (host only): dict with the Q
    brick (t, y, x), the pairing axis, units and KV steps per head."""
    qb = (ctypes.c_int * 4)()
    units, steps = ctypes.c_longlong(0), ctypes.c_longlong(0)
    _check(lib.dit_na3d_plan(T, Y, X, Kt, Ky, Kx, qb, ctypes.byref(units), ctypes.byref(steps)), "dit_na3d_plan")
    return {"q_brick": (qb[0], qb[1], qb[2]), "pair_axis": qb[3], "units_per_head": units.value,
            "steps_per_head": steps.value}


def neighborhood_attention(q, k, v, grid, kernel, scale: Optional[float] = None, with_lse: bool = True,
                           stream=None):
    """(out bf16, lse fp32 or None) of 3-D neighborhood attention; q, k, v [B,H,T*Y*X,D] bf16,
    grid = (T, Y, X), kernel = (Kt, Ky, Kx)."""
    import torch
    B, H, S, D = _dims(q)
    scale = (1.0 / D ** 0.5) if scale is None else scale
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if with_lse else None
    dit_na3d_fwd(q, k, v, out, lse, B, H, *grid, D, *kernel, scale, stream)
    return out, lse


def dit_swap01_chunks(src, dst, d0: int, d1: int, chunk_bytes: int, stream=None) -> None:
    _check(lib.dit_swap01_chunks(_ptr(src), _ptr(dst), int(d0), int(d1), int(chunk_bytes), _stream(stream)),
           "dit_swap01_chunks")


def dit_quant_fp8_blocks(x_bf16, x_fp8, descales, B: int, H: int, S: int, D: int, stream=None) -> None:
    _check(lib.dit_quant_fp8_blocks(_ptr(x_bf16), _ptr(x_fp8), _ptr(descales), B, H, S, D, _stream(stream)),
           "dit_quant_fp8_blocks")


def dit_attn_fwd_fp8_blocks(q8, k8, v8, dq_blk, dk_blk, dv_blk, out, lse, B: int, H: int, S_q: int, S_kv: int,
                            D: int, k0: int, k1: int, scale: float, out_dtype: int = 0, stream=None) -> None:
    _check(lib.dit_attn_fwd_fp8_blocks(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(dq_blk), _ptr(dk_blk), _ptr(dv_blk),
                                       _ptr(out), _ptr(lse), B, H, S_q, S_kv, D, k0, k1, float(scale), out_dtype,
                                       _stream(stream)), "dit_attn_fwd_fp8_blocks")


def dit_quant_fp8_noalloc(x_bf16, x_fp8, descale, n: int, stream=None) -> None:
    """dit_quant_fp8 without a workspace, for callers that cannot allocate device memory
    (the scratch is a small array inside the library's device data; see the header)."""
    _check(lib.dit_quant_fp8_noalloc(_ptr(x_bf16), _ptr(x_fp8), _ptr(descale), int(n), _stream(stream)),
           "dit_quant_fp8_noalloc")


def dit_device_status(clear: bool = True) -> int:
    st = ctypes.c_int(0)
    _check(lib.dit_device_status(ctypes.byref(st), 1 if clear else 0), "dit_device_status")
    return st.value


def dit_set_wait_timeout_us(us: int) -> None:
    _check(lib.dit_set_wait_timeout_us(int(us)), "dit_set_wait_timeout_us")


def dit_set_sm_reserve(n_sms: int) -> None:
    _check(lib.dit_set_sm_reserve(int(n_sms)), "dit_set_sm_reserve")


def dit_selftest_wait_timeout(timeout_us: int, stream=None) -> None:
    _check(lib.dit_selftest_wait_timeout(int(timeout_us), _stream(stream)), "dit_selftest_wait_timeout")


def dit_version() -> int:
    return int(lib.dit_version())


# --------------------------------------------------------------------------- torch helpers

def _dims(q):
    if q.dim() != 4:
        raise ValueError("expected a [B, H, S, D] tensor")
    return tuple(int(x) for x in q.shape)


def attention(q, k, v, scale: Optional[float] = None, with_lse: bool = True, descale_qkv=None,
              stream=None) -> Tuple[object, Optional[object]]:
    """out (bf16) and lse (fp32) of full attention; q/k/v bf16 or uint8 E4M3 codes."""
    import torch
    B, H, S, D = _dims(q)
    fp8 = q.dtype == torch.uint8
    scale = (1.0 / D ** 0.5) if scale is None else scale
    out = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if with_lse else None
    dit_attn_fwd(q, k, v, out, lse, B, H, S, D, scale, DIT_FP8_E4M3 if fp8 else DIT_BF16, descale_qkv, stream)
    return out, lse


def attention_chunk(q, k, v, k0: int, k1: int, scale: Optional[float] = None, out_dtype=None,
                    descale_qkv=None, stream=None):
    """Partial (out, lse) over keys [k0, k1); out fp32 unless out_dtype is torch.bfloat16."""
    import torch
    B, H, S_q, D = _dims(q)
    S_kv = int(k.shape[2])
    fp8 = q.dtype == torch.uint8
    scale = (1.0 / D ** 0.5) if scale is None else scale
    od = torch.float32 if out_dtype is None else out_dtype
    out = torch.empty((B, H, S_q, D), dtype=od, device=q.device)
    lse = torch.empty((B, H, S_q), dtype=torch.float32, device=q.device)
    dit_attn_fwd_chunk(q, k, v, out, lse, B, H, S_q, S_kv, D, k0, k1, scale,
                       DIT_FP8_E4M3 if fp8 else DIT_BF16, DIT_FP32 if od == torch.float32 else DIT_BF16,
                       descale_qkv, stream)
    return out, lse


def ring_attention(q, k, v, bounds: Sequence, scale: Optional[float] = None, descale_qkv=None, stream=None):
    """Attention accumulated over the KV ranges in `bounds` with fused ring steps:
    (out fp32, lse) = exact attention over the union of the ranges."""
    import torch
    B, H, S_q, D = _dims(q)
    S_kv = int(k.shape[2])
    fp8 = q.dtype == torch.uint8
    scale = (1.0 / D ** 0.5) if scale is None else scale
    out = torch.empty((B, H, S_q, D), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, S_q), dtype=torch.float32, device=q.device)
    dit_attn_acc_init(out, lse, B, H, S_q, D, stream)
    for k0, k1 in bounds:
        dit_attn_fwd_chunk_acc(q, k, v, out, lse, B, H, S_q, S_kv, D, k0, k1, scale,
                               DIT_FP8_E4M3 if fp8 else DIT_BF16, descale_qkv, stream)
    return out, lse


def merge(outs: Sequence, lses: Sequence, out_dtype=None, stream=None):
    """Merged (out, lse) of chunk partials; out bf16 unless out_dtype is torch.float32."""
    import torch
    B, H, S, D = _dims(outs[0])
    od = torch.bfloat16 if out_dtype is None else out_dtype
    out = torch.empty((B, H, S, D), dtype=od, device=outs[0].device)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=outs[0].device)
    in_dt = DIT_FP32 if outs[0].dtype == torch.float32 else DIT_BF16
    dit_attn_merge(outs, lses, out, lse, B, H, S, D, in_dt, DIT_FP32 if od == torch.float32 else DIT_BF16, stream)
    return out, lse


def quantize_fp8_blocks(x, stream=None):
    """(codes uint8 [B,H,S,D], descales fp32 [B,H,ceil(S/128)]) of a bf16 [B,H,S,D] tensor."""
    import torch
    B, H, S, D = _dims(x)
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    ds = torch.empty((B, H, (S + 127) // 128), dtype=torch.float32, device=x.device)
    dit_quant_fp8_blocks(x, codes, ds, B, H, S, D, stream)
    return codes, ds


def attention_fp8_blocks(q8, k8, v8, dq, dk, dv, scale: Optional[float] = None, k0: int = 0, k1: Optional[int] = None,
                         out_dtype=None, stream=None):
    """(out, lse) of E4M3 inputs with per-block descales over keys [k0, k1)."""
    import torch
    B, H, S_q, D = _dims(q8)
    S_kv = int(k8.shape[2])
    k1 = S_kv if k1 is None else k1
    scale = (1.0 / D ** 0.5) if scale is None else scale
    odt = torch.bfloat16 if out_dtype is None else out_dtype
    out = torch.empty((B, H, S_q, D), dtype=odt, device=q8.device)
    lse = torch.empty((B, H, S_q), dtype=torch.float32, device=q8.device)
    dit_attn_fwd_fp8_blocks(q8, k8, v8, dq, dk, dv, out, lse, B, H, S_q, S_kv, D, k0, k1, scale,
                            DIT_FP32 if odt == torch.float32 else DIT_BF16, stream)
    return out, lse


def quantize_fp8(x, stream=None):
    """(codes uint8 same shape, descale fp32 [1]) of a bf16 tensor; per-tensor absmax scale."""
    import torch
    n = x.numel()
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    descale = torch.empty((1,), dtype=torch.float32, device=x.device)
    ws_bytes = dit_quant_fp8_workspace_bytes(n)
    ws = torch.empty((ws_bytes // 4,), dtype=torch.float32, device=x.device)
    dit_quant_fp8(x, codes, descale, n, ws, ws_bytes, stream)
    return codes, descale
