"""Dynamic Bifocal RoPE attention (Jet-Long) for NVIDIA B200, sm_100a.

Thin Python binding over the C ABI of ``lib/libbifocal.so`` (declared in
include/bifocal.h). Every step of the attention path runs in the library's CUDA
kernels; this module only marshals arguments: it takes torch tensors for device
memory, allocates outputs and workspace through torch, passes raw pointers and the
current CUDA stream, and turns a non-zero status into ``BifocalError``. There is no
CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

__all__ = [
    "BifocalError", "FREQ_INTERP", "POS_ALIAS", "FLAG_FORCE_BIFOCAL", "FLAG_MMA_SYNC", "FLAG_WINDOW", "FLAG_FUSED_ROPE", "Params", "lib", "lib_path",
    "bifocal_factor", "bifocal_prefill", "bifocal_prefill_rope", "bifocal_prefill_attention", "rope_causal_prefill", "bifocal_prefill_chunk_paged", "bifocal_decode", "bifocal_decode_noalloc", "rope_causal_decode",
    "prefill_workspace_size", "decode_workspace_size", "last_device_error", "build_info", "test_set_fault",
    "STATUS_TIMEOUT", "STATUS_RANGE", "STATUS_INDEX", "FAULT_NONE", "FAULT_PREFILL_SKIP_FILL", "FAULT_DECODE_SKIP_STAGE",
]

FREQ_INTERP = "freq_interp"
POS_ALIAS = "pos_alias"
_MODES = {FREQ_INTERP: 0, POS_ALIAS: 1}
FLAG_FORCE_BIFOCAL = 1
FLAG_MMA_SYNC = 2
FLAG_WINDOW = 4
FLAG_FUSED_ROPE = 8
DTYPE_BF16, DTYPE_FP32 = 0, 1
STATUS_TIMEOUT, STATUS_RANGE, STATUS_INDEX = 4, 7, 8
FAULT_NONE, FAULT_PREFILL_SKIP_FILL, FAULT_DECODE_SKIP_STAGE = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.path.join(_HERE, "lib", "libbifocal.so")


class BifocalError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().bifocal_status_string(status).decode() if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})")


class Params(ctypes.Structure):
    _fields_ = [
        ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("w0", ctypes.c_int32),
        ("w_pretrained", ctypes.c_int32), ("mode", ctypes.c_int32), ("rope_theta", ctypes.c_double),
        ("softmax_scale", ctypes.c_float), ("flags", ctypes.c_int32),
    ]


_LIB: Optional[ctypes.CDLL] = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise ImportError(f"libbifocal.so is not built ({path}); run "
                              "`python -m rope_context_extension_bifocal_b200.build`")
        L = ctypes.CDLL(path)
        vp, i32, sz, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_int64
        pp = ctypes.POINTER(Params)
        L.bifocal_factor.argtypes, L.bifocal_factor.restype = [i64, i32], i32
        L.bifocal_prefill_workspace_size.argtypes = [i32, i32, i32, pp]
        L.bifocal_prefill_workspace_size.restype = sz
        L.bifocal_decode_workspace_size.argtypes, L.bifocal_decode_workspace_size.restype = [i32, pp], sz
        pre = [vp, vp, vp, i32, i32, i32, pp, vp, vp, vp, vp, vp, sz, vp]
        for name in ("bifocal_prefill", "rope_causal_prefill"):
            getattr(L, name).argtypes, getattr(L, name).restype = pre, i32
        L.bifocal_prefill_rope.argtypes = [vp, vp, vp, i32, i32, i32, pp, vp, vp, vp, sz, vp]
        L.bifocal_prefill_rope.restype = i32
        L.bifocal_prefill_rope_qknorm.argtypes = [vp, vp, vp, i32, i32, i32, pp, vp, vp, ctypes.c_float, vp, vp,
                                                  vp, sz, vp]
        L.bifocal_prefill_rope_qknorm.restype = i32
        L.bifocal_prefill_attention.argtypes = [vp, i32, i32, i32, pp, vp, vp, vp, sz, vp]
        L.bifocal_prefill_attention.restype = i32
        L.bifocal_prefill_chunk_workspace_size.argtypes = [i32, i32, pp]
        L.bifocal_prefill_chunk_workspace_size.restype = sz
        L.bifocal_prefill_chunk.argtypes = [vp, vp, vp, i32, i32, i32, pp, vp, vp, i32, vp, vp, vp, sz, vp]
        L.bifocal_prefill_chunk.restype = i32
        dec = [vp, vp, vp, vp, vp, i32, i32, pp, vp, vp, vp, sz, vp]
        for name in ("bifocal_decode", "rope_causal_decode"):
            getattr(L, name).argtypes, getattr(L, name).restype = dec, i32
        L.bifocal_decode_paged_workspace_size.argtypes = [i32, i32, pp]
        L.bifocal_decode_paged_workspace_size.restype = sz
        L.bifocal_decode_paged.argtypes = [vp, vp, vp, vp, vp, i32, i32, vp, i32, vp, i32, i32, pp, vp, vp, vp, sz,
                                           vp]
        L.bifocal_decode_paged.restype = i32
        L.bifocal_prefill_chunk_paged.argtypes = [vp, vp, vp, i32, vp, vp, pp, vp, vp, i32, i32, vp, i32, vp, vp,
                                                  vp]
        L.bifocal_prefill_chunk_paged.restype = i32
        L.bifocal_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, pp, vp, vp, vp]
        L.bifocal_decode_noalloc.restype = i32
        L.bifocal_status_string.argtypes, L.bifocal_status_string.restype = [i32], ctypes.c_char_p
        L.bifocal_last_device_error.argtypes, L.bifocal_last_device_error.restype = [vp], i32
        L.bifocal_build_info.argtypes, L.bifocal_build_info.restype = [], ctypes.c_char_p
        L.bifocal_device_status_word.argtypes, L.bifocal_device_status_word.restype = [], i32
        L.bifocal_test_set_fault.argtypes, L.bifocal_test_set_fault.restype = [i32, i32, i64], i32
        _LIB = L
    return _LIB


def lib() -> ctypes.CDLL:
    """The loaded C library (raises ImportError when it is not built)."""
    return _lib()


def build_info() -> str:
    return _lib().bifocal_build_info().decode()


def bifocal_factor(L: int, w_pretrained: int) -> int:
    """G = max(1, ceil(L / w_pretrained)), computed by the library."""
    g = _lib().bifocal_factor(int(L), int(w_pretrained))
    if g < 0:
        raise BifocalError(1, "bifocal_factor")
    return g


def make_params(hq, hkv, head_dim, w0=0, w_pretrained=1, theta=10000.0, mode=FREQ_INTERP, scale=None, flags=0):
    return Params(int(hq), int(hkv), int(head_dim), int(w0), int(w_pretrained), _MODES[mode], float(theta),
                  0.0 if scale is None else float(scale), int(flags))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise BifocalError(status, where)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_FP32
    raise BifocalError(2, f"unsupported dtype {t.dtype}")


def prefill_workspace_size(dtype, batch, L, params: Params) -> int:
    return int(_lib().bifocal_prefill_workspace_size(dtype, batch, L, ctypes.byref(params)))


def decode_workspace_size(L_max, params: Params) -> int:
    return int(_lib().bifocal_decode_workspace_size(L_max, ctypes.byref(params)))


def _workspace(nbytes: int, device):
    import torch
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _prefill(fn_name, q, k, v, params, want_lse, want_cache, out, workspace, stream):
    import torch
    b, L, hq, D = q.shape
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous():
            raise BifocalError(1, f"{fn_name}: q, k, v must be contiguous CUDA tensors")
    dt = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise BifocalError(1, f"{fn_name}: q, k, v must share a dtype")
    out = torch.empty(b, L, hq, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(b, hq, L, dtype=torch.float32, device=q.device) if want_lse else None
    kc = vc = None
    if want_cache:
        kc = torch.empty(b, L, k.shape[2], D, dtype=torch.bfloat16, device=q.device)
        vc = torch.empty_like(kc)
    need = prefill_workspace_size(dt, b, L, params)
    ws = _workspace(need, q.device) if workspace is None else workspace
    st = getattr(_lib(), fn_name)(_ptr(q), _ptr(k), _ptr(v), dt, b, L, ctypes.byref(params), _ptr(out), _ptr(lse),
                                  _ptr(kc), _ptr(vc), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, fn_name)
    return out, lse, kc, vc


def bifocal_prefill(q, k, v, *, w0: int, w_pretrained: int, theta: float, mode: str = FREQ_INTERP,
                    scale: Optional[float] = None, flags: int = 0, want_lse: bool = True,
                    want_cache: bool = False, out=None, workspace=None, stream=None):
    """Bifocal causal prefill. q [b, L, Hq, D], k and v [b, L, Hkv, D] raw (bf16 or fp32), on CUDA.

    Returns (out [b, L, Hq, D] bf16, lse [b, Hq, L] fp32 or None, kcache, vcache or None).
    """
    p = make_params(q.shape[2], k.shape[2], q.shape[3], w0, w_pretrained, theta, mode, scale, flags)
    return _prefill("bifocal_prefill", q, k, v, p, want_lse, want_cache, out, workspace, stream)


def bifocal_prefill_rope(q, k, v, params: Params, workspace, kcache=None, vcache=None, stream=None):
    """Step 1 of bifocal_prefill: the RoPE pass into `workspace` (see include/bifocal.h)."""
    st = _lib().bifocal_prefill_rope(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), q.shape[0], q.shape[1],
                                     ctypes.byref(params), _ptr(kcache), _ptr(vcache), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bifocal_prefill_rope")


def bifocal_prefill_rope_qknorm(q, k, v, params: Params, workspace, q_norm_w, k_norm_w, eps: float = 1e-6,
                                kcache=None, vcache=None, stream=None):
    """Step 1 with Qwen3's per-head q/k RMS norm fused in (weights [D], input dtype)."""
    st = _lib().bifocal_prefill_rope_qknorm(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), q.shape[0], q.shape[1],
                                            ctypes.byref(params), _ptr(q_norm_w), _ptr(k_norm_w), float(eps),
                                            _ptr(kcache), _ptr(vcache), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bifocal_prefill_rope_qknorm")


def bifocal_prefill_attention(v, params: Params, workspace, out, lse=None, batch=None, L=None, dtype=None,
                              stream=None):
    """Step 2 of bifocal_prefill: the fused attention over the operands step 1 left in `workspace`."""
    b = out.shape[0] if batch is None else batch
    n = out.shape[1] if L is None else L
    dt = _dtype_code(v) if dtype is None else dtype
    st = _lib().bifocal_prefill_attention(_ptr(v), dt, b, n, ctypes.byref(params), _ptr(out), _ptr(lse),
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream(stream))
    _check(st, "bifocal_prefill_attention")


def rope_causal_prefill(q, k, v, *, theta: float, scale: Optional[float] = None, want_lse: bool = True,
                        want_cache: bool = False, out=None, workspace=None, stream=None):
    """Plain causal attention under the original RoPE (the comparator)."""
    p = make_params(q.shape[2], k.shape[2], q.shape[3], 0, 1, theta, FREQ_INTERP, scale, 0)
    return _prefill("rope_causal_prefill", q, k, v, p, want_lse, want_cache, out, workspace, stream)


def prefill_chunk_workspace_size(P0: int, C: int, params: Params) -> int:
    return int(_lib().bifocal_prefill_chunk_workspace_size(int(P0), int(C), ctypes.byref(params)))


def bifocal_prefill_chunk(q, k, v, kcache, vcache, P0: int, *, w0: int, w_pretrained: int, theta: float,
                          mode: str = FREQ_INTERP, scale: Optional[float] = None, flags: int = 0,
                          want_lse: bool = True, out=None, workspace=None, stream=None):
    """Chunked prefill over a cache (batch 1). q [C, Hq, D], k / v [C, Hkv, D] raw (bf16 or fp32) at
    positions P0..P0+C-1; kcache / vcache [cap, Hkv, D] bf16 hold P0 cached rows (original-RoPE keys)
    and receive the chunk's rows. Returns (out [C, Hq, D] bf16, lse [Hq, C] fp32 or None)."""
    import torch
    C, hq, D = q.shape
    p = make_params(hq, k.shape[1], D, w0, w_pretrained, theta, mode, scale, flags)
    out = torch.empty(C, hq, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(hq, C, dtype=torch.float32, device=q.device) if want_lse else None
    need = prefill_chunk_workspace_size(P0, C, p)
    ws = _workspace(need, q.device) if workspace is None else workspace
    st = _lib().bifocal_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), int(P0), int(C), ctypes.byref(p),
                                      _ptr(kcache), _ptr(vcache), kcache.shape[0], _ptr(out), _ptr(lse), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bifocal_prefill_chunk")
    return out, lse


def bifocal_prefill_chunk_paged(q, k, v, chunk_lens, cached_lens, kpool, vpool, page_size: int, block_table, *,
                                w0: int, w_pretrained: int, theta: float, mode: str = FREQ_INTERP,
                                scale: Optional[float] = None, flags: int = 0, want_lse: bool = True, out=None,
                                stream=None):
    """Chunked prefill for a batch over a paged cache. q [T, Hq, D], k / v [T, Hkv, D] raw bf16, the
    chunks packed in batch order; chunk_lens / cached_lens: Python ints per sequence; kpool / vpool
    [pages * page_size, Hkv, D] bf16; block_table [B, max_pages] int32 on the device. Returns
    (out [T, Hq, D] bf16, lse [Hq, T] fp32 or None)."""
    import torch
    T, hq, D = q.shape
    B = len(chunk_lens)
    if len(cached_lens) != B or sum(int(c) for c in chunk_lens) != T:
        raise BifocalError(1, "bifocal_prefill_chunk_paged: chunk_lens must sum to the packed rows")
    p = make_params(hq, k.shape[1], D, w0, w_pretrained, theta, mode, scale, flags)
    out = torch.empty(T, hq, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(hq, T, dtype=torch.float32, device=q.device) if want_lse else None
    cl = (ctypes.c_int32 * B)(*[int(c) for c in chunk_lens])
    pl = (ctypes.c_int32 * B)(*[int(c) for c in cached_lens])
    st = _lib().bifocal_prefill_chunk_paged(_ptr(q), _ptr(k), _ptr(v), B, cl, pl, ctypes.byref(p), _ptr(kpool),
                                            _ptr(vpool), kpool.shape[0] // page_size, int(page_size),
                                            _ptr(block_table), block_table.shape[1], _ptr(out), _ptr(lse),
                                            _stream(stream))
    _check(st, "bifocal_prefill_chunk_paged")
    return out, lse


def _decode(fn_name, q, k_new, v_new, kcache, vcache, L, params, want_lse, out, workspace, stream):
    import torch
    hq, D = q.shape
    cap = kcache.shape[0]
    out = torch.empty(hq, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(hq, dtype=torch.float32, device=q.device) if want_lse else None
    ws = _workspace(decode_workspace_size(L, params), q.device) if workspace is None else workspace
    st = getattr(_lib(), fn_name)(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kcache), _ptr(vcache), cap, int(L),
                                  ctypes.byref(params), _ptr(out), _ptr(lse), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    _check(st, fn_name)
    return out, lse


def bifocal_decode(q, k_new, v_new, kcache, vcache, L: int, *, w0: int, w_pretrained: int, theta: float,
                   mode: str = FREQ_INTERP, scale: Optional[float] = None, flags: int = 0, want_lse: bool = True,
                   out=None, workspace=None, stream=None):
    """One decode step at length L (including the new token). q [Hq, D], k_new / v_new [Hkv, D] raw bf16;
    kcache / vcache [cap, Hkv, D] bf16 (original-RoPE keys); row L-1 is written. Returns (out, lse)."""
    p = make_params(q.shape[0], k_new.shape[0], q.shape[1], w0, w_pretrained, theta, mode, scale, flags)
    return _decode("bifocal_decode", q, k_new, v_new, kcache, vcache, L, p, want_lse, out, workspace, stream)


def bifocal_decode_noalloc(q, k_new, v_new, kcache, vcache, L: int, *, w0: int, w_pretrained: int, theta: float,
                           mode: str = FREQ_INTERP, scale: Optional[float] = None, flags: int = 0,
                           want_lse: bool = True, out=None, lse=None, stream=None):
    """bifocal_decode with the library's static scratch instead of a workspace.

    For callers that cannot allocate device memory themselves. Pass preallocated `out`
    (and `lse`) to keep the call itself free of allocations; calls that overlap on the GPU
    share the scratch and race (see include/bifocal.h)."""
    import torch
    hq, D = q.shape
    p = make_params(hq, k_new.shape[0], D, w0, w_pretrained, theta, mode, scale, flags)
    out = torch.empty(hq, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty(hq, dtype=torch.float32, device=q.device)
    st = _lib().bifocal_decode_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kcache), _ptr(vcache),
                                       kcache.shape[0], int(L), ctypes.byref(p), _ptr(out),
                                       _ptr(lse if want_lse else None), _stream(stream))
    _check(st, "bifocal_decode_noalloc")
    return out, (lse if want_lse else None)


def decode_paged_workspace_size(batch: int, max_len: int, params: Params) -> int:
    return int(_lib().bifocal_decode_paged_workspace_size(int(batch), int(max_len), ctypes.byref(params)))


def bifocal_decode_paged(q, k_new, v_new, kpool, vpool, page_size: int, block_table, seq_lens, max_len: int, *,
                         w0: int, w_pretrained: int, theta: float, mode: str = FREQ_INTERP,
                         scale: Optional[float] = None, flags: int = 0, want_lse: bool = True, out=None,
                         workspace=None, stream=None):
    """Batched decode over a paged cache. q [B, Hq, D], k_new / v_new [B, Hkv, D] bf16; kpool / vpool
    [pages * page_size, Hkv, D] bf16; block_table [B, max_pages] int32 and seq_lens [B] int32 on the
    device (lengths with the new token); max_len bounds them. Returns (out [B, Hq, D], lse [B, Hq])."""
    import torch
    B, hq, D = q.shape
    p = make_params(hq, k_new.shape[1], D, w0, w_pretrained, theta, mode, scale, flags)
    out = torch.empty(B, hq, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(B, hq, dtype=torch.float32, device=q.device) if want_lse else None
    ws = _workspace(decode_paged_workspace_size(B, max_len, p), q.device) if workspace is None else workspace
    pool_pages = kpool.shape[0] // page_size
    st = _lib().bifocal_decode_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kpool), _ptr(vpool), pool_pages,
                                     int(page_size), _ptr(block_table), block_table.shape[1], _ptr(seq_lens),
                                     int(max_len), B, ctypes.byref(p), _ptr(out), _ptr(lse), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bifocal_decode_paged")
    return out, lse


def rope_causal_decode(q, k_new, v_new, kcache, vcache, L: int, *, theta: float, scale: Optional[float] = None,
                       want_lse: bool = True, out=None, workspace=None, stream=None):
    p = make_params(q.shape[0], k_new.shape[0], q.shape[1], 0, 1, theta, FREQ_INTERP, scale, 0)
    return _decode("rope_causal_decode", q, k_new, v_new, kcache, vcache, L, p, want_lse, out, workspace, stream)


def device_status_word() -> int:
    """Raw device status word: 0, or code | (site << 8) of the first device-side event (code 1: a
    bounded wait expired, 2: an fp16 operand out of range, 3: a device-side index out of range)."""
    return int(_lib().bifocal_device_status_word())


def last_device_error(stream=None) -> int:
    """Status of the device-side checks since the last call, then cleared: 0, STATUS_TIMEOUT (a
    bounded wait expired), STATUS_RANGE (an fp16 QK^T operand was out of range) or STATUS_INDEX (a
    sequence length or block-table entry in device memory was out of range)."""
    return int(_lib().bifocal_last_device_error(_stream(stream)))


def test_set_fault(kind: int = FAULT_NONE, arg: int = 0, wait_limit_ns: int = 0) -> None:
    """Test-only fault injection (see bifocal_test_set_fault in include/bifocal.h); the default
    arguments turn every injection off and restore the 2 s wait limit."""
    _check(_lib().bifocal_test_set_fault(int(kind), int(arg), int(wait_limit_ns)), "bifocal_test_set_fault")
