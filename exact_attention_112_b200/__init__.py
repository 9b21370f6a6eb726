"""B200-native (sm_100a) exact scaled dot-product attention behind a C ABI.

The compute lives in ``libfa.so`` (CUDA for sm_100a: TMA, tcgen05 tensor cores,
tensor memory; see ``include/fa.h``).  This module only marshals arguments:
it turns torch tensors into device pointers and sizes, calls the C entry point
of the same name and raises ``FaError`` on a non-zero status.  There is no
fallback: if the library is missing or the device is not an sm_100 GPU the
calls fail.

    import exact_attention_112_b200 as fa
    o, lse = fa.attention_forward(q, k, v, causal=True)         # allocates o, lse
    fa.fa_fwd(q, k, v, o, lse, causal=True, scale=None)          # caller-owned outputs
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, dO, causal=True)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

__all__ = [
    "FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA",
    "FA_ERR_DEVICE_TIMEOUT", "FA_ERR_WORKSPACE", "FA_ERR_INTERNAL", "FA_F16", "FA_BF16", "FaError",
    "lib", "library_path", "fa_fwd", "fa_fwd_fp8", "fa_bwd", "fa_bwd_workspace_bytes",
    "fa_bwd_noalloc",
    "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_bytes", "fa_splitkv_num_splits", "fa_fwd_mask", "fa_bwd_mask",
    "fa_fwd_varlen", "fa_bwd_varlen", "fa_mask_tile_flags_bytes", "mask_tile_flags",
    "FA_BWD_NOALLOC_MAX_ROWS",
    "fa_status_string", "fa_device_status", "fa_debug_wait_timeout", "fa_launch_count",
    "fa_profile_enable", "fa_profile_read",
    "attention_forward", "attention_backward",
]

(FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_DEVICE_TIMEOUT,
 FA_ERR_WORKSPACE, FA_ERR_INTERNAL) = range(7)
FA_F16, FA_BF16 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return os.path.join(_HERE, "libfa.so")


class FaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {fa_status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with "
                    "`python -m exact_attention_112_b200._build` (needs nvcc)")
            L = ctypes.CDLL(path)
            vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp]
            L.fa_fwd.restype = i
            L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, f, f, vp, vp]
            L.fa_fwd_fp8.restype = i
            ll = ctypes.c_longlong
            L.fa_fwd_mask.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, i, i, ll, vp, vp]
            L.fa_fwd_mask.restype = i
            L.fa_bwd_mask.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i,
                                      vp, i, i, ll, vp, vp, sz, vp]
            L.fa_bwd_mask.restype = i
            L.fa_mask_tile_flags_bytes.argtypes = [i, i, i, i]
            L.fa_mask_tile_flags_bytes.restype = sz
            L.fa_mask_tile_flags.argtypes = [vp, i, i, i, i, ll, vp, sz, vp]
            L.fa_mask_tile_flags.restype = i
            L.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, i, vp]
            L.fa_fwd_varlen.restype = i
            L.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                        i, i, f, i, vp, sz, vp]
            L.fa_bwd_varlen.restype = i
            L.fa_fwd_splitkv_workspace_bytes.argtypes = [i, i, i, i, i, i]
            L.fa_fwd_splitkv_workspace_bytes.restype = sz
            L.fa_splitkv_num_splits.argtypes = [i, i, i, i, i]
            L.fa_splitkv_num_splits.restype = i
            L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, i, vp, sz, vp]
            L.fa_fwd_splitkv.restype = i
            L.fa_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
            L.fa_bwd_workspace_bytes.restype = sz
            L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i,
                                 vp, vp, sz, vp]
            L.fa_bwd.restype = i
            L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f,
                                         i, vp, vp]
            L.fa_bwd_noalloc.restype = i
            L.fa_status_string.argtypes = [i]
            L.fa_status_string.restype = ctypes.c_char_p
            L.fa_device_status.argtypes = [vp]
            L.fa_device_status.restype = i
            L.fa_profile_enable.argtypes = [i]
            L.fa_profile_enable.restype = i
            L.fa_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float),
                                          ctypes.POINTER(ctypes.c_char_p), i,
                                          ctypes.POINTER(ctypes.c_int)]
            L.fa_profile_read.restype = i
            L.fa_launch_count.argtypes = []
            L.fa_launch_count.restype = ctypes.c_ulonglong
            L.fa_debug_wait_timeout.argtypes = [ctypes.c_uint, vp]
            L.fa_debug_wait_timeout.restype = i
            _lib = L
    return _lib


def fa_status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.float16:
        return FA_F16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise FaError(FA_ERR_UNSUPPORTED, f"dtype {t.dtype}")


def _check(status, what):
    if status != FA_OK:
        raise FaError(status, what)


def _bad(what, msg):
    raise FaError(FA_ERR_INVALID_ARG, f"{what}: {msg}")


def _validate(what, q, k, v, *, o=None, lse=None, dO=None, dq=None, dk=None, dv=None,
              key_bias=None, workspace=None, outputs=(), fp8=False):
    """Check every tensor handed to the C ABI before its pointer is taken.

    The library sees only pointers and the sizes derived from ``q`` and ``k``,
    so a tensor of the wrong shape, dtype, layout or device would make the
    kernels read or write outside its allocation.  Checked here: q is
    [B,H,Nq,D] f16/bf16; k, v are [B,H,Nk,D] of q's dtype; o, dO, dq have q's
    shape and dtype; dk, dv have k's; lse is float32 [B,H,Nq]; key_bias is
    float32 [B,Nk]; every tensor (workspace included) is contiguous and on the
    current CUDA device.  With ``fp8``, q, k, v are float8_e4m3fn and o is
    bf16.  Returns (B, H, Nq, Nk, D, dtype code).
    """
    import torch
    if q is None or q.dim() != 4:
        _bad(what, "q must be a 4-D tensor [B, H, Nq, D]")
    if fp8:
        if q.dtype != torch.float8_e4m3fn:
            raise FaError(FA_ERR_UNSUPPORTED, f"{what}: q must be torch.float8_e4m3fn, got {q.dtype}")
        code, out_dt = None, torch.bfloat16
    else:
        code = _dtype_code(q)
        out_dt = q.dtype
    B, H, Nq, D = q.shape
    if k is None or v is None:
        _bad(what, "k and v are required")
    if k.dim() != 4 or tuple(k.shape[:2]) != (B, H) or k.shape[3] != D:
        _bad(what, f"k must be [B={B}, H={H}, Nk, D={D}], got {tuple(k.shape)}")
    Nk = k.shape[2]
    want = {"q": (q, (B, H, Nq, D), q.dtype), "k": (k, (B, H, Nk, D), q.dtype),
            "v": (v, (B, H, Nk, D), q.dtype)}
    for name, t, shape, dt in (("o", o, (B, H, Nq, D), out_dt),
                               ("lse", lse, (B, H, Nq), torch.float32),
                               ("dO", dO, (B, H, Nq, D), q.dtype),
                               ("dq", dq, (B, H, Nq, D), q.dtype),
                               ("dk", dk, (B, H, Nk, D), q.dtype),
                               ("dv", dv, (B, H, Nk, D), q.dtype),
                               ("key_bias", key_bias, (B, Nk), torch.float32)):
        if t is not None:
            want[name] = (t, shape, dt)
        elif name in outputs:
            _bad(what, f"{name} is required")
    for name, (t, shape, dt) in want.items():
        if tuple(t.shape) != shape:
            _bad(what, f"{name} must have shape {shape}, got {tuple(t.shape)}")
        if t.dtype != dt:
            _bad(what, f"{name} must be {dt}, got {t.dtype}")
    tensors = [t for t, _, _ in want.values()]
    if workspace is not None:
        tensors.append(workspace)
    for t in tensors:
        if not t.is_contiguous():
            _bad(what, "every tensor must be contiguous")
    for t in tensors:
        if not t.is_cuda:
            _bad(what, f"every tensor must be on a CUDA device, got {t.device}")
    dev = torch.cuda.current_device()
    for t in tensors:
        if t.device.index != dev:
            _bad(what, f"every tensor must be on the current device cuda:{dev}, got {t.device}")
    return B, H, Nq, Nk, D, code


def fa_fwd(q, k, v, o, lse, causal=False, scale=None, key_bias=None, stream=None):
    """Forward pass into caller-owned ``o`` [B,H,Nq,D] and ``lse`` [B,H,Nq] fp32."""
    B, H, Nq, Nk, D, code = _validate("fa_fwd", q, k, v, o=o, lse=lse, key_bias=key_bias,
                                      outputs=("o", "lse"))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    st = lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, D,
                      int(bool(causal)), float(scale), code, _ptr(key_bias),
                      _stream_ptr(stream))
    _check(st, "fa_fwd")


def fa_fwd_fp8(q, k, v, o, lse, causal=False, scale=None, q_descale=1.0, k_descale=1.0,
               v_descale=1.0, key_bias=None, stream=None):
    """FP8 forward: q, k, v float8_e4m3fn [B,H,N,128] standing for
    q_descale*q, k_descale*k, v_descale*v; writes bf16 ``o`` and fp32 ``lse``."""
    B, H, Nq, Nk, D, _ = _validate("fa_fwd_fp8", q, k, v, o=o, lse=lse, key_bias=key_bias,
                                   outputs=("o", "lse"), fp8=True)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    st = lib().fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, D,
                          int(bool(causal)), float(scale), float(q_descale), float(k_descale),
                          float(v_descale), _ptr(key_bias), _stream_ptr(stream))
    _check(st, "fa_fwd_fp8")


def _mask_args(what, mask, B, H, Nq, Nk, device):
    """(mask_B, mask_H, ldm) of a general additive mask tensor: float32 of shape
    [B or 1, H or 1, Nq, Nk] (or [Nq, Nk]) whose rows are contiguous and whose
    row stride ldm is a multiple of 4 elements (a view of a [.., .., Nq, ldm]
    buffer with ldm >= Nk is accepted), on the given device."""
    import torch
    if mask is None:
        _bad(what, "mask is required")
    m = mask if mask.dim() == 4 else mask.reshape(1, 1, *mask.shape) if mask.dim() == 2 else None
    if m is None or tuple(m.shape[2:]) != (Nq, Nk) or m.shape[0] not in (1, B) or m.shape[1] not in (1, H):
        _bad(what, f"mask must have shape [B or 1, H or 1, {Nq}, {Nk}], got {tuple(mask.shape)}")
    if m.dtype != torch.float32:
        _bad(what, f"mask must be torch.float32, got {m.dtype}")
    Bm, Hm = int(m.shape[0]), int(m.shape[1])
    ldm = int(m.stride(2)) if Nq > 1 else max(4, (Nk + 3) // 4 * 4)
    if Nk > 0 and m.stride(3) != 1:
        _bad(what, "mask rows must be contiguous")
    if ldm < Nk or ldm % 4 != 0 or ldm < 4:
        _bad(what, f"mask row stride must be >= Nk and a multiple of 4 elements, got {ldm}")
    if (Hm > 1 and m.stride(1) != Nq * ldm) or (Bm > 1 and m.stride(0) != Hm * Nq * ldm):
        _bad(what, "mask planes must be stored one after another")
    if not m.is_cuda or m.device != device:
        _bad(what, f"mask must be on {device}, got {m.device}")
    if m.data_ptr() % 16 != 0:
        _bad(what, "mask must start 16-byte aligned")
    return Bm, Hm, ldm


def _flags_arg(what, flags, Bm, Hm, Nq, Nk, device):
    """A mask tile summary must be a contiguous uint8 tensor of
    fa_mask_tile_flags_bytes() elements on the mask's device (or None)."""
    import torch
    if flags is None:
        return None
    need = fa_mask_tile_flags_bytes(Bm, Hm, Nq, Nk)
    if flags.dtype != torch.uint8 or not flags.is_contiguous() or flags.numel() != need:
        _bad(what, f"tile_flags must be a contiguous uint8 tensor of {need} elements")
    if not flags.is_cuda or flags.device != device:
        _bad(what, f"tile_flags must be on {device}")
    return flags


def fa_mask_tile_flags_bytes(mask_B, mask_H, Nq, Nk) -> int:
    return int(lib().fa_mask_tile_flags_bytes(mask_B, mask_H, Nq, Nk))


def mask_tile_flags(mask, Nq=None, Nk=None, stream=None):
    """Tile summary of a general mask (see include/fa.h, fa_mask_tile_flags):
    a uint8 tensor [planes, ceil(Nq/128), ceil(Nk/128)], 1 where a 128 x 128
    tile has an entry above -inf."""
    import torch
    m = mask if mask.dim() == 4 else mask.reshape(1, 1, *mask.shape)
    Bm, Hm, Nq_, Nk_ = (int(x) for x in m.shape)
    Bm, Hm, ldm = _mask_args("fa_mask_tile_flags", mask, Bm, Hm, Nq_, Nk_, mask.device)
    out = torch.empty((Bm * Hm, (Nq_ + 127) // 128, (Nk_ + 127) // 128), dtype=torch.uint8,
                      device=mask.device)
    st = lib().fa_mask_tile_flags(_ptr(mask), Bm, Hm, Nq_, Nk_, ldm, _ptr(out), out.numel(),
                                  _stream_ptr(stream))
    _check(st, "fa_mask_tile_flags")
    return out


def fa_fwd_mask(q, k, v, o, lse, mask, causal=False, scale=None, tile_flags=None, stream=None):
    """Forward with a general additive mask (see include/fa.h); tile_flags is
    the optional summary from mask_tile_flags()."""
    B, H, Nq, Nk, D, code = _validate("fa_fwd_mask", q, k, v, o=o, lse=lse, outputs=("o", "lse"))
    Bm, Hm, ldm = _mask_args("fa_fwd_mask", mask, B, H, Nq, Nk, q.device)
    flags = _flags_arg("fa_fwd_mask", tile_flags, Bm, Hm, Nq, Nk, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    st = lib().fa_fwd_mask(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, D,
                           int(bool(causal)), float(scale), code, _ptr(mask), Bm, Hm, ldm,
                           _ptr(flags), _stream_ptr(stream))
    _check(st, "fa_fwd_mask")


def fa_bwd_mask(q, k, v, o, lse, dO, dq, dk, dv, workspace, mask, causal=False, scale=None,
                tile_flags=None, stream=None):
    """Backward with a general additive mask (see include/fa.h); tile_flags is
    the optional summary from mask_tile_flags()."""
    B, H, Nq, Nk, D, code = _validate("fa_bwd_mask", q, k, v, o=o, lse=lse, dO=dO, dq=dq, dk=dk,
                                      dv=dv, workspace=workspace,
                                      outputs=("o", "lse", "dO", "dq", "dk", "dv"))
    Bm, Hm, ldm = _mask_args("fa_bwd_mask", mask, B, H, Nq, Nk, q.device)
    flags = _flags_arg("fa_bwd_mask", tile_flags, Bm, Hm, Nq, Nk, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    nbytes = workspace.numel() * workspace.element_size()
    st = lib().fa_bwd_mask(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                           _ptr(dk), _ptr(dv), B, H, Nq, Nk, D, int(bool(causal)), float(scale),
                           code, _ptr(mask), Bm, Hm, ldm, _ptr(flags), _ptr(workspace), nbytes,
                           _stream_ptr(stream))
    _check(st, "fa_bwd_mask")


def _varlen_args(what, q, k, cu_q, cu_k, max_q, max_k):
    """Shapes of the packed layout: q [H, total_q, D], k [H, total_k, D], the
    int32 sequence tables [num_seqs + 1] on q's device."""
    import torch
    if q is None or q.dim() != 3 or k is None or k.dim() != 3:
        _bad(what, "packed q and k must be 3-D tensors [H, total, D]")
    H, total_q, D = q.shape
    if k.shape[0] != H or k.shape[2] != D:
        _bad(what, f"k must be [H={H}, total_k, D={D}], got {tuple(k.shape)}")
    for name, t in (("cu_seqlens_q", cu_q), ("cu_seqlens_k", cu_k)):
        if t is None or t.dim() != 1 or t.dtype != torch.int32 or not t.is_contiguous():
            _bad(what, f"{name} must be a contiguous int32 vector [num_seqs + 1]")
        if not t.is_cuda or t.device != q.device:
            _bad(what, f"{name} must be on {q.device}")
    if cu_q.numel() != cu_k.numel() or cu_q.numel() < 2:
        _bad(what, "cu_seqlens_q and cu_seqlens_k must both have num_seqs + 1 >= 2 entries")
    if int(max_q) < 0 or int(max_k) < 0:
        _bad(what, "max_seqlen_q and max_seqlen_k must be >= 0")
    return int(cu_q.numel() - 1), H, total_q, int(k.shape[1]), D


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                  causal=False, scale=None, stream=None):
    """Forward of packed variable-length sequences (see include/fa.h): q, o
    [H, total_q, D], k, v [H, total_k, D], lse [H, total_q]."""
    nseq, H, tq, tk, D = _varlen_args("fa_fwd_varlen", q, k, cu_seqlens_q, cu_seqlens_k,
                                      max_seqlen_q, max_seqlen_k)
    # the packed tensors are the fixed layout with B = 1 and N = total
    _, _, _, _, _, code = _validate("fa_fwd_varlen", q[None], k[None], v[None] if v is not None else None,
                                    o=None if o is None else o[None],
                                    lse=None if lse is None else lse[None], outputs=("o", "lse"))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    st = lib().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                             _ptr(cu_seqlens_k), nseq, H, tq, tk, int(max_seqlen_q),
                             int(max_seqlen_k), D, int(bool(causal)), float(scale), code,
                             _stream_ptr(stream))
    _check(st, "fa_fwd_varlen")


def fa_bwd_varlen(q, k, v, o, lse, dO, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k,
                  max_seqlen_q, max_seqlen_k, causal=False, scale=None, stream=None):
    """Backward of packed variable-length sequences (see include/fa.h)."""
    nseq, H, tq, tk, D = _varlen_args("fa_bwd_varlen", q, k, cu_seqlens_q, cu_seqlens_k,
                                      max_seqlen_q, max_seqlen_k)
    add = lambda t: None if t is None else t[None]
    _, _, _, _, _, code = _validate("fa_bwd_varlen", q[None], k[None], add(v), o=add(o), lse=add(lse),
                                    dO=add(dO), dq=add(dq), dk=add(dk), dv=add(dv),
                                    workspace=workspace,
                                    outputs=("o", "lse", "dO", "dq", "dk", "dv"))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    nbytes = workspace.numel() * workspace.element_size()
    st = lib().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                             _ptr(dk), _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), nseq, H,
                             tq, tk, int(max_seqlen_q), int(max_seqlen_k), D, int(bool(causal)),
                             float(scale), code, _ptr(workspace), nbytes, _stream_ptr(stream))
    _check(st, "fa_bwd_varlen")


def fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, D, num_splits) -> int:
    return int(lib().fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, D, num_splits))


def fa_splitkv_num_splits(B, H, Nq, Nk, num_sms=0) -> int:
    """A num_splits for fa_fwd_splitkv on these sizes (num_sms 0: the current
    device's SM count)."""
    return int(lib().fa_splitkv_num_splits(B, H, Nq, Nk, num_sms))


def fa_fwd_splitkv(q, k, v, o, lse, num_splits, workspace, causal=False, scale=None,
                   key_bias=None, stream=None):
    """Split-KV forward (few queries, many keys) into caller-owned o, lse,
    with a caller-owned workspace of fa_fwd_splitkv_workspace_bytes() bytes."""
    B, H, Nq, Nk, D, code = _validate("fa_fwd_splitkv", q, k, v, o=o, lse=lse,
                                      key_bias=key_bias, workspace=workspace,
                                      outputs=("o", "lse"))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    nbytes = workspace.numel() * workspace.element_size()
    st = lib().fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, D,
                              int(bool(causal)), float(scale), code, _ptr(key_bias),
                              int(num_splits), _ptr(workspace), nbytes, _stream_ptr(stream))
    _check(st, "fa_fwd_splitkv")


def fa_bwd_workspace_bytes(B, H, Nq, Nk, D) -> int:
    return int(lib().fa_bwd_workspace_bytes(B, H, Nq, Nk, D))


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, workspace, causal=False, scale=None,
           key_bias=None, stream=None):
    """Backward pass into caller-owned dq, dk, dv, using a caller-owned workspace."""
    B, H, Nq, Nk, D, code = _validate("fa_bwd", q, k, v, o=o, lse=lse, dO=dO, dq=dq, dk=dk,
                                      dv=dv, key_bias=key_bias, workspace=workspace,
                                      outputs=("o", "lse", "dO", "dq", "dk", "dv"))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    nbytes = workspace.numel() * workspace.element_size()
    st = lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                      _ptr(dk), _ptr(dv), B, H, Nq, Nk, D, int(bool(causal)), float(scale),
                      code, _ptr(key_bias), _ptr(workspace), nbytes,
                      _stream_ptr(stream))
    _check(st, "fa_bwd")


def _header_define(name: str) -> int:
    """Integer value of a ``#define`` in include/fa.h (the one source of the
    library's compile-time limits)."""
    import re
    path = os.path.join(os.path.dirname(_HERE), "include", "fa.h")
    with open(path) as f:
        m = re.search(rf"^#define\s+{name}\s+(\d+)\s*$", f.read(), flags=re.M)
    if m is None:
        raise RuntimeError(f"{name} is not defined in {path}")
    return int(m.group(1))


FA_BWD_NOALLOC_MAX_ROWS = _header_define("FA_BWD_NOALLOC_MAX_ROWS")


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, causal=False, scale=None, key_bias=None,
                   stream=None):
    """Backward without a workspace, for callers that cannot allocate device
    memory (the scratch is a fixed array inside libfa.so; B*H*Nq must not
    exceed FA_BWD_NOALLOC_MAX_ROWS).  See include/fa.h."""
    B, H, Nq, Nk, D, code = _validate("fa_bwd_noalloc", q, k, v, o=o, lse=lse, dO=dO, dq=dq,
                                      dk=dk, dv=dv, key_bias=key_bias,
                                      outputs=("o", "lse", "dO", "dq", "dk", "dv"))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    st = lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                              _ptr(dk), _ptr(dv), B, H, Nq, Nk, D, int(bool(causal)),
                              float(scale), code, _ptr(key_bias), _stream_ptr(stream))
    _check(st, "fa_bwd_noalloc")


def fa_device_status(stream=None) -> int:
    return int(lib().fa_device_status(_stream_ptr(stream)))


def fa_profile_enable(on: bool = True) -> None:
    _check(lib().fa_profile_enable(int(bool(on))), "fa_profile_enable")


def fa_profile_read(capacity: int = 4096):
    """[(kernel name, milliseconds), ...] of the launches recorded since the
    last read on this thread (see fa_profile_enable)."""
    ms = (ctypes.c_float * capacity)()
    names = (ctypes.c_char_p * capacity)()
    n = ctypes.c_int(0)
    _check(lib().fa_profile_read(ms, names, capacity, ctypes.byref(n)), "fa_profile_read")
    return [(names[i].decode(), float(ms[i])) for i in range(n.value)]


def fa_launch_count() -> int:
    return int(lib().fa_launch_count())


def fa_debug_wait_timeout(timeout_us: int, stream=None) -> int:
    return int(lib().fa_debug_wait_timeout(int(timeout_us), _stream_ptr(stream)))


def attention_forward(q, k, v, causal=False, scale=None, key_bias=None, stream=None):
    """Allocate O and LSE with torch (device plumbing) and run ``fa_fwd``."""
    import torch
    B, H, Nq, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, o, lse, causal=causal, scale=scale, key_bias=key_bias, stream=stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dO, causal=False, scale=None, key_bias=None,
                       stream=None):
    """Allocate dq, dk, dv and the workspace with torch and run ``fa_bwd``."""
    import torch
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ws = torch.empty(fa_bwd_workspace_bytes(B, H, Nq, Nk, D), dtype=torch.uint8, device=q.device)
    fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, ws, causal=causal, scale=scale,
           key_bias=key_bias, stream=stream)
    return dq, dk, dv
