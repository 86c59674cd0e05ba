"""Python binding of libfa_sm100.so (exact attention for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/fa.h. PyTorch supplies device
memory and the current stream. There is no CPU fallback: if the library is
missing, every call raises.

Functions carry the C names:
    fa_fwd, fa_fwd_ex, fa_fwd_f32, fa_fwd_tf32, fa_fp8_prepare, fa_fwd_fp8, fa_fp8_vt_keys,
    fa_bwd_ex,
    fa_bwd, fa_bwd_workspace_size,
    fa_decode_splitkv, fa_decode_workspace_size,
    fa_device_status, fa_set_wait_limit, fa_debug_skip_load
"""
from __future__ import annotations

import ctypes
import math
import os
import re

__all__ = [
    "FAError", "library_path", "load_library", "exported_symbols",
    "fa_fwd", "fa_fwd_pair", "fa_fwd_ex", "fa_bwd_ex", "fa_dropout_keep_threshold", "fa_fwd_f32", "fa_fwd_tf32", "fa_fp8_prepare", "fa_fwd_fp8",
    "fa_fp8_vt_keys",
    "fa_bwd", "fa_bwd_workspace_size",
    "fa_decode_splitkv", "fa_decode_workspace_size", "fa_decode_splitkv_static",
    "fa_decode_paged",
    "fa_device_status",
    "fa_set_wait_limit", "fa_debug_skip_load", "fa_abi_version",
    "fa_profile_begin", "fa_profile_end", "STATUS", "KERNEL_NAMES",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

STATUS = {
    0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED",
    3: "FA_ERR_ALIGNMENT", 4: "FA_ERR_WORKSPACE", 5: "FA_ERR_CUDA",
    6: "FA_ERR_TIMEOUT",
}


class FAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libfa_sm100.so")


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t

_SIGNATURES = {
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_last_error": (ctypes.c_char_p, []),
    "fa_abi_version": (_I, []),
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_tf32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_pair": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, ctypes.c_longlong,
                       ctypes.c_longlong, _F, ctypes.c_ulonglong, ctypes.c_uint, _P]),
    "fa_bwd_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P,
                       ctypes.c_longlong, ctypes.c_longlong, _F, ctypes.c_ulonglong, ctypes.c_uint,
                       _P, _S, _P]),
    "fa_fp8_vt_keys": (_I, [_I]),
    "fa_dropout_keep_threshold": (_I, [_F]),
    "fa_fp8_prepare": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_workspace_size": (_S, [_I, _I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I,
                    _P, _S, _P]),
    "fa_decode_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "fa_decode_splitkv": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I,
                               _P, _S, _P]),
    "fa_decode_splitkv_static": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                             _P, _S, _P]),
    "fa_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint)]),
    "fa_set_wait_limit": (None, [ctypes.c_ulonglong]),
    "fa_debug_skip_load": (None, [_I]),
    "fa_profile_begin": (None, []),
    "fa_profile_end": (_I, [ctypes.POINTER(_I), ctypes.POINTER(ctypes.c_double), _I]),
}

KERNEL_NAMES = {1: "fwd", 2: "fwd_f32", 3: "bwd_pre", 4: "bwd_dkdv", 5: "bwd_dq",
                6: "decode_split", 7: "decode_merge", 9: "fp8_prep"}


def load_library():
    """Load libfa_sm100.so; raise if it has not been built."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with "
                "`python -m exact_attention_130_b200.build` (there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def exported_symbols():
    """Names of the entry points include/fa.h declares."""
    hdr = open(os.path.join(os.path.dirname(_HERE), "include", "fa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(fa_\w+)\s*\(", hdr, re.M)))


def _check(status: int):
    if status != 0:
        lib = load_library()
        raise FAError(status, lib.fa_last_error().decode(errors="replace"))


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fa_abi_version() -> int:
    return load_library().fa_abi_version()


def fa_fwd(q, k, v, causal: bool = False, scale: float | None = None, o=None,
           lse=None, stream=None):
    """O, LSE = attention(q, k, v); bf16 [B, H, N, d] in and out."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    _check(lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                      scale, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_fwd_pair(q, k, v, causal: bool = False, scale: float | None = None, o=None,
                lse=None, stream=None):
    """fa_fwd on pairs of CTAs sharing each tensor-core product (d = 128)."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    _check(lib.fa_fwd_pair(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                           scale, int(bool(causal)), _stream(stream)))
    return o, lse


def _bias_args(bias, B, H, N):
    """(pointer, stride_b, stride_h) of a bf16 bias broadcastable to [B, H, N, N]."""
    import torch
    if bias is None:
        return None, 0, 0
    if bias.dtype != torch.bfloat16 or not bias.is_cuda:
        raise TypeError("bias must be a bf16 CUDA tensor")
    if bias.dim() != 4 or bias.shape[-2:] != (N, N) or bias.shape[0] not in (1, B) \
            or bias.shape[1] not in (1, H):
        raise ValueError("bias must have shape [B or 1, H or 1, N, N]")
    if bias.stride(3) != 1 or bias.stride(2) != N:
        raise ValueError("bias rows must be contiguous")
    sb = bias.stride(0) if bias.shape[0] > 1 else 0
    sh = bias.stride(1) if bias.shape[1] > 1 else 0
    return _ptr(bias), sb, sh


def fa_fwd_ex(q, k, v, causal: bool = False, scale: float | None = None, bias=None,
              p_drop: float = 0.0, seed: int = 0, offset: int = 0, o=None, lse=None,
              stream=None):
    """fa_fwd with an additive bf16 bias [B|1, H|1, N, N] and dropout on P
    (Philox4x32-10 keyed by ``seed``, sequence ``offset``)."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    bp, sb, sh = _bias_args(bias, B, H, N)
    _check(lib.fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, scale,
                         int(bool(causal)), bp, sb, sh, float(p_drop), int(seed), int(offset),
                         _stream(stream)))
    return o, lse


def fa_dropout_keep_threshold(p_drop: float) -> int:
    """The keep threshold t of fa_fwd_ex / fa_bwd_ex for p_drop (-1 if invalid)."""
    return int(load_library().fa_dropout_keep_threshold(float(p_drop)))


def fa_bwd_ex(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None, bias=None,
              p_drop: float = 0.0, seed: int = 0, offset: int = 0, dq=None, dk=None, dv=None,
              workspace=None, stream=None):
    """fa_bwd for fa_fwd_ex (same bias, p_drop, seed and offset)."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    bp, sb, sh = _bias_args(bias, B, H, N)
    _check(lib.fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                         _ptr(dk), _ptr(dv), B, H, N, d, scale, int(bool(causal)), bp, sb, sh,
                         float(p_drop), int(seed), int(offset), _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream(stream)))
    return dq, dk, dv


def fa_fwd_f32(q, k, v, causal: bool = False, scale: float | None = None,
               o=None, lse=None, stream=None):
    """The fp32 forward: fp32 [B, H, N, d] in and out."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.float32, n)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check(lib.fa_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N,
                          d, scale, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_fwd_tf32(q, k, v, causal: bool = False, scale: float | None = None,
               o=None, lse=None, stream=None):
    """fa_fwd_f32 with both products on the tensor cores in TF32 (inputs
    rounded to TF32 to nearest): faster, errors ~1e-4 to 1e-3."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.float32, n)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check(lib.fa_fwd_tf32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N,
                          d, scale, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_fp8_vt_keys(N: int) -> int:
    """Keys per row of the transposed V codes (N rounded up to 16)."""
    return int(load_library().fa_fp8_vt_keys(N))


def fa_fp8_prepare(q, k, v, signs=None, out=None, stream=None):
    """Rotate (when ``signs`` is given) and quantise bf16 q, k, v
    [B, H, N, 128] to e4m3 codes for ``fa_fwd_fp8``. Returns a dict with
    q8, k8 (uint8 [B, H, N, 128]), vt8 (uint8 [B, H, 128, fa_fp8_vt_keys(N)]),
    q_scale, k_scale (fp32 [B, H, ceil(N / 128)]) and v_amax (fp32 [B, H]);
    ``out`` may supply those tensors."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    if signs is not None:
        _need(signs, torch.float32, "signs")
        if signs.numel() != d:
            raise ValueError("signs must hold d entries")
    nb = (N + 127) // 128
    dev = q.device
    if out is None:
        u8 = torch.uint8
        out = {
            "q8": torch.empty((B, H, N, d), dtype=u8, device=dev),
            "k8": torch.empty((B, H, N, d), dtype=u8, device=dev),
            "vt8": torch.empty((B, H, d, max(fa_fp8_vt_keys(N), 1)), dtype=u8, device=dev),
            "q_scale": torch.empty((B, H, nb), dtype=torch.float32, device=dev),
            "k_scale": torch.empty((B, H, nb), dtype=torch.float32, device=dev),
            "v_amax": torch.empty((B, H), dtype=torch.float32, device=dev),
        }
    for n in ("q8", "k8", "vt8"):
        _need(out[n], torch.uint8, n)
    for n in ("q_scale", "k_scale", "v_amax"):
        _need(out[n], torch.float32, n)
    _check(lib.fa_fp8_prepare(_ptr(q), _ptr(k), _ptr(v), _ptr(signs) if signs is not None else None,
                              B, H, N, d, _ptr(out["q8"]), _ptr(out["k8"]), _ptr(out["vt8"]),
                              _ptr(out["q_scale"]), _ptr(out["k_scale"]), _ptr(out["v_amax"]),
                              _stream(stream)))
    return out


def fa_fwd_fp8(prep, causal: bool = False, scale: float | None = None, o=None, lse=None,
               stream=None):
    """O (bf16), LSE = attention of the FP8 operands that ``fa_fp8_prepare``
    made (``scale`` applies to the original Q K^T, default 1/sqrt(d))."""
    import torch
    lib = load_library()
    q8 = prep["q8"]
    B, H, N, d = q8.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o is None:
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    _check(lib.fa_fwd_fp8(_ptr(q8), _ptr(prep["k8"]), _ptr(prep["vt8"]), _ptr(prep["q_scale"]),
                          _ptr(prep["k_scale"]), _ptr(prep["v_amax"]), _ptr(o), _ptr(lse),
                          B, H, N, d, scale, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None,
           dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of sum(O * dO); bf16 tensors, fp32 lse."""
    import torch
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do),
                      _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, scale,
                      int(bool(causal)), _ptr(workspace), workspace.numel(),
                      _stream(stream)))
    return dq, dk, dv


def fa_decode_workspace_size(B: int, H: int, Lmax: int, d: int,
                             num_splits: int = 0) -> int:
    return int(load_library().fa_decode_workspace_size(B, H, Lmax, d, num_splits))


def fa_decode_splitkv(q, kcache, vcache, seqlens, scale: float | None = None,
                      num_splits: int = 0, o=None, lse=None, workspace=None,
                      stream=None):
    """Single-token attention over a KV cache, split-KV with LSE merge."""
    import torch
    lib = load_library()
    _need(q, torch.bfloat16, "q")
    _need(kcache, torch.bfloat16, "kcache")
    _need(vcache, torch.bfloat16, "vcache")
    _need(seqlens, torch.int32, "seqlens")
    B, H, d = q.shape
    Lmax = kcache.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    need = fa_decode_workspace_size(B, H, Lmax, d, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(lib.fa_decode_splitkv(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens),
                                 _ptr(o), _ptr(lse), B, H, Lmax, d, scale,
                                 num_splits, _ptr(workspace), workspace.numel(),
                                 _stream(stream)))
    return o, lse


def fa_decode_paged(q, kpages, vpages, block_table, seqlens, scale: float | None = None,
                    num_splits: int = 0, o=None, lse=None, workspace=None, stream=None):
    """Single-token attention over a paged KV cache with grouped query heads.

    q [B, Hq, d]; kpages, vpages [num_pages, Hkv, page_size, d];
    block_table int32 [B, max_pages]; seqlens int32 [B] (all on the device).
    """
    import torch
    lib = load_library()
    _need(q, torch.bfloat16, "q")
    _need(kpages, torch.bfloat16, "kpages")
    _need(vpages, torch.bfloat16, "vpages")
    _need(block_table, torch.int32, "block_table")
    _need(seqlens, torch.int32, "seqlens")
    B, Hq, d = q.shape
    num_pages, Hkv, page_size = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    max_pages = block_table.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    need = fa_decode_workspace_size(B, Hq, max_pages * page_size, d, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(lib.fa_decode_paged(_ptr(q), _ptr(kpages), _ptr(vpages), _ptr(block_table),
                               _ptr(seqlens), _ptr(o), _ptr(lse), B, Hq, Hkv, num_pages,
                               page_size, max_pages, d, scale, num_splits, _ptr(workspace),
                               workspace.numel(), _stream(stream)))
    return o, lse


def fa_decode_splitkv_static(q, kcache, vcache, seqlens, scale: float | None = None,
                             num_splits: int = 0, o=None, lse=None, stream=None):
    """fa_decode_splitkv with the partials in the library's own 8 MiB device
    buffer: for callers that cannot allocate device memory while decoding.
    Calls that may overlap on the GPU share that buffer and must be
    serialised by the caller."""
    import torch
    lib = load_library()
    _need(q, torch.bfloat16, "q")
    _need(kcache, torch.bfloat16, "kcache")
    _need(vcache, torch.bfloat16, "vcache")
    _need(seqlens, torch.int32, "seqlens")
    B, H, d = q.shape
    Lmax = kcache.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(lib.fa_decode_splitkv_static(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens),
                                        _ptr(o), _ptr(lse), B, H, Lmax, d, scale,
                                        num_splits, _stream(stream)))
    return o, lse


def fa_device_status(stream=None):
    """Synchronise the stream; return (status, raw word) of the device."""
    lib = load_library()
    word = ctypes.c_uint(0)
    st = lib.fa_device_status(_stream(stream), ctypes.byref(word))
    return st, word.value


def fa_set_wait_limit(nanoseconds: int):
    load_library().fa_set_wait_limit(int(nanoseconds))


def fa_debug_skip_load(kernel=True):
    """Test hook: the next call leaves one load out of the named kernel.

    `kernel` is a kernel id or a name from KERNEL_NAMES ("fwd", "bwd_dkdv",
    "bwd_dq", "decode_split"); True means the forward, False or 0 clears.
    """
    if isinstance(kernel, str):
        ids = {name: kid for kid, name in KERNEL_NAMES.items()}
        if kernel not in ids:
            raise ValueError(f"unknown kernel name {kernel!r}")
        kid = ids[kernel]
    else:
        kid = int(kernel)
    load_library().fa_debug_skip_load(kid)


def fa_profile_begin():
    load_library().fa_profile_begin()


def fa_profile_end():
    """Stop per-kernel timing; return {kernel name: (launches, total ms)}."""
    lib = load_library()
    launches = (ctypes.c_int * 16)()
    total = (ctypes.c_double * 16)()
    rc = lib.fa_profile_end(launches, total, 16)
    if rc < 0:
        raise FAError(5, "fa_profile_end: a CUDA event call failed")
    return {KERNEL_NAMES[k]: (launches[k], total[k]) for k in KERNEL_NAMES if launches[k]}
