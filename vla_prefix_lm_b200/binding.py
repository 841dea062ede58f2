"""ctypes binding of libpiattn.so for torch tensors: argument marshalling only.

Every computation happens in the CUDA library; this module checks that the
tensors it is handed match the ABI's layout (device, dtype, contiguity),
fills the descriptor, passes raw pointers and the current CUDA stream, and
turns a non-zero status into an exception.  There is no fallback: if the
library cannot be loaded, every call raises.

Names mirror the C ABI in include/pi_attn.h: ``pi_attn_prefill``,
``pi_attn_suffix``, ``pi_attn_suffix_workspace_bytes``, ``pi_attn_debug_mask``,
``pi_attn_read_status``, ``pi_attn_set_wait_limit``, ``pi_attn_selftest_wait``.
"""

from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpiattn.so")

PI_BF16, PI_F32 = 0, 1
PI_OK, PI_ERR_ARG, PI_ERR_ALIGN, PI_ERR_UNSUPPORTED, PI_ERR_CUDA, PI_ERR_TIMEOUT = range(6)

EXPORTED = (
    "pi_attn_prefill",
    "pi_attn_suffix",
    "pi_attn_suffix_workspace_bytes",
    "pi_attn_debug_mask",
    "pi_attn_read_status",
    "pi_attn_status_string",
    "pi_attn_set_wait_limit",
    "pi_attn_selftest_wait",
    "pi_attn_suffix_masked",
    "pi_attn_suffix_noalloc",
    "pi_rope_inplace",
    "pi_euler_update",
    "pi_attn_prefill_backward",
    "pi_attn_prefill_backward_workspace_bytes",
    "pi_attn_suffix_noalloc_capacity",
    "pi_attn_debug_tiles",
    "pi_attn_prefill_ws",
    "pi_attn_prefill_workspace_bytes",
    "pi_attn_prefill_tail_splits",
)


class PiAttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


class PiRopeDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32),
        ("S", ctypes.c_int32),
        ("P", ctypes.c_int32),
        ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("base", ctypes.c_float),
        ("mask_batch_stride", ctypes.c_int64),
        ("prefix_batch_stride", ctypes.c_int64),
    ]


class PiAttnDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32),
        ("Sq", ctypes.c_int32),
        ("P", ctypes.c_int32),
        ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("mask_batch_stride", ctypes.c_int64),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libpiattn.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m vla_prefix_lm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        dp = ctypes.POINTER(PiAttnDesc)
        L.pi_attn_prefill.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.pi_attn_prefill.restype = i32
        L.pi_attn_prefill_ws.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.pi_attn_prefill_ws.restype = i32
        L.pi_attn_prefill_workspace_bytes.argtypes = [dp]
        L.pi_attn_prefill_workspace_bytes.restype = sz
        L.pi_attn_prefill_tail_splits.argtypes = [dp]
        L.pi_attn_prefill_tail_splits.restype = i32
        L.pi_attn_suffix.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.pi_attn_suffix.restype = i32
        L.pi_attn_suffix_workspace_bytes.argtypes = [dp]
        L.pi_attn_suffix_workspace_bytes.restype = sz
        L.pi_attn_debug_mask.argtypes = [dp, i32, vp, vp, vp, vp]
        L.pi_attn_debug_mask.restype = i32
        L.pi_attn_read_status.argtypes = [vp]
        L.pi_attn_read_status.restype = i32
        L.pi_attn_status_string.argtypes = [i32]
        L.pi_attn_status_string.restype = ctypes.c_char_p
        L.pi_attn_set_wait_limit.argtypes = [ctypes.c_uint64]
        L.pi_attn_set_wait_limit.restype = ctypes.c_uint64
        L.pi_attn_debug_tiles.argtypes = [dp, vp, vp, vp, vp]
        L.pi_attn_debug_tiles.restype = i32
        L.pi_attn_selftest_wait.argtypes = [vp]
        L.pi_attn_selftest_wait.restype = i32
        L.pi_attn_suffix_masked.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.pi_attn_suffix_masked.restype = i32
        L.pi_rope_inplace.argtypes = [ctypes.POINTER(PiRopeDesc), vp, vp, vp, vp, vp, vp]
        L.pi_rope_inplace.restype = i32
        L.pi_euler_update.argtypes = [vp, vp, i32, ctypes.c_float, ctypes.c_int64, vp]
        L.pi_euler_update.restype = i32
        L.pi_attn_suffix_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.pi_attn_suffix_noalloc.restype = i32
        L.pi_attn_prefill_backward_workspace_bytes.argtypes = [dp]
        L.pi_attn_prefill_backward_workspace_bytes.restype = sz
        L.pi_attn_prefill_backward.argtypes = [dp] + [vp] * 12 + [sz, vp]
        L.pi_attn_prefill_backward.restype = i32
        L.pi_attn_suffix_noalloc_capacity.argtypes = []
        L.pi_attn_suffix_noalloc_capacity.restype = sz
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().pi_attn_status_string(int(code)).decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, name, dtype=None, dims=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got {t.dim()}")


def _mask_stride(ar, B, S):
    if ar.dim() == 1:
        if ar.shape[0] != S:
            raise ValueError(f"ar_mask has {ar.shape[0]} tokens, expected {S}")
        return 0
    if ar.dim() == 2 and ar.shape == (B, S):
        return S
    raise ValueError(f"ar_mask must be [S] or [B, S], got {tuple(ar.shape)}")


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return PI_BF16
    if t.dtype == torch.float32:
        return PI_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def pi_attn_prefill_workspace_bytes(q, k, ar_mask, softmax_scale=1.0):
    """Bytes of the scratch pi_attn_prefill takes as ``workspace`` (0: this
    geometry does not use one)."""
    B, S, Hq, d = q.shape
    desc = PiAttnDesc(B, S, 0, Hq, k.shape[2], d, _dtype_code(q), float(softmax_scale),
                      _mask_stride(ar_mask, B, S))
    return int(lib().pi_attn_prefill_workspace_bytes(ctypes.byref(desc)))


def pi_attn_prefill_tail_splits(q, k, ar_mask, softmax_scale=1.0):
    """Pieces per last-round query tile a call with a workspace splits into on
    this device (1: none, one kernel launch per call; else two)."""
    B, S, Hq, d = q.shape
    desc = PiAttnDesc(B, S, 0, Hq, k.shape[2], d, _dtype_code(q), float(softmax_scale),
                      _mask_stride(ar_mask, B, S))
    return int(lib().pi_attn_prefill_tail_splits(ctypes.byref(desc)))


def pi_attn_prefill(q, k, v, ar_mask, segment_ids=None, out=None, lse=None,
                    softmax_scale=1.0, stream=None, workspace=None):
    """Joint prefill.  q [B,S,Hq,d]; k, v [B,S,Hkv,d]; ar_mask uint8 [S] or [B,S];
    segment_ids int32 like ar_mask or None.  Returns ``out`` (allocated if None).
    ``workspace``: a CUDA byte tensor of pi_attn_prefill_workspace_bytes bytes
    (lets a sparse last round of query tiles split over idle SM pairs), or None."""
    _need(q, "q", dims=4)
    _need(k, "k", q.dtype, 4)
    _need(v, "v", q.dtype, 4)
    _need(ar_mask, "ar_mask", torch.uint8)
    B, S, Hq, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[1] != S or k.shape[3] != d:
        raise ValueError("k/v shape mismatch")
    mbs = _mask_stride(ar_mask, B, S)
    if segment_ids is not None:
        _need(segment_ids, "segment_ids", torch.int32)
        if segment_ids.shape != ar_mask.shape:
            raise ValueError("segment_ids must have ar_mask's shape")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, 4)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    desc = PiAttnDesc(B, S, 0, Hq, k.shape[2], d, _dtype_code(q), float(softmax_scale), mbs)
    if workspace is None:
        rc = lib().pi_attn_prefill(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(ar_mask), _ptr(segment_ids), _ptr(out), _ptr(lse),
                                   ctypes.c_void_p(_stream(stream)))
    else:
        _need(workspace, "workspace", torch.uint8)
        rc = lib().pi_attn_prefill_ws(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(ar_mask), _ptr(segment_ids), _ptr(out), _ptr(lse),
                                      _ptr(workspace), workspace.numel(),
                                      ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        raise PiAttnError(rc, "pi_attn_prefill")
    return out


def pi_attn_prefill_backward_workspace_bytes(q, k, ar_mask, softmax_scale=1.0):
    B, S, Hq, d = q.shape
    desc = PiAttnDesc(B, S, 0, Hq, k.shape[2], d, _dtype_code(q), float(softmax_scale),
                      _mask_stride(ar_mask, B, S))
    return int(lib().pi_attn_prefill_backward_workspace_bytes(ctypes.byref(desc)))


def pi_attn_prefill_backward(q, k, v, ar_mask, out, lse, dout, segment_ids=None, dq=None,
                             dk=None, dv=None, workspace=None, softmax_scale=1.0, stream=None):
    """Gradient of pi_attn_prefill: (dq, dk, dv) in fp32, allocated if None.
    ``out`` and ``lse`` are the forward's outputs for the same inputs; ``dout``
    has q's dtype and shape.  ``workspace``: a CUDA uint8 tensor of at least
    pi_attn_prefill_backward_workspace_bytes (allocated here if None)."""
    _need(q, "q", dims=4)
    _need(k, "k", q.dtype, 4)
    _need(v, "v", q.dtype, 4)
    _need(out, "out", q.dtype, 4)
    _need(dout, "dout", q.dtype, 4)
    _need(lse, "lse", torch.float32)
    _need(ar_mask, "ar_mask", torch.uint8)
    B, S, Hq, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[1] != S or k.shape[3] != d:
        raise ValueError("k/v shape mismatch")
    if out.shape != q.shape or dout.shape != q.shape or tuple(lse.shape) != (B, S, Hq):
        raise ValueError("out/dout must have q's shape and lse must be [B, S, Hq]")
    mbs = _mask_stride(ar_mask, B, S)
    if segment_ids is not None:
        _need(segment_ids, "segment_ids", torch.int32)
        if segment_ids.shape != ar_mask.shape:
            raise ValueError("segment_ids must have ar_mask's shape")
    desc = PiAttnDesc(B, S, 0, Hq, k.shape[2], d, _dtype_code(q), float(softmax_scale), mbs)
    need = int(lib().pi_attn_prefill_backward_workspace_bytes(ctypes.byref(desc)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    f32 = torch.float32
    dq = torch.empty(q.shape, dtype=f32, device=q.device) if dq is None else dq
    dk = torch.empty(k.shape, dtype=f32, device=q.device) if dk is None else dk
    dv = torch.empty(v.shape, dtype=f32, device=q.device) if dv is None else dv
    _need(dq, "dq", f32, 4)
    _need(dk, "dk", f32, 4)
    _need(dv, "dv", f32, 4)
    if dq.shape != q.shape or dk.shape != k.shape or dv.shape != v.shape:
        raise ValueError("dq/dk/dv must have the shapes of q/k/v")
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().pi_attn_prefill_backward(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(ar_mask), _ptr(segment_ids),
        _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
        ws_bytes, ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        raise PiAttnError(rc, "pi_attn_prefill_backward")
    return dq, dk, dv


def _suffix_desc(q_suf, k_suf, k_cache, ar_mask_suf, softmax_scale):
    B, Sq, Hq, d = q_suf.shape
    P = 0 if k_cache is None else k_cache.shape[1]
    mbs = _mask_stride(ar_mask_suf, B, Sq)
    return PiAttnDesc(B, Sq, P, Hq, k_suf.shape[2], d, _dtype_code(q_suf),
                      float(softmax_scale), mbs)


def pi_attn_suffix_workspace_bytes(q_suf, k_suf, k_cache, ar_mask_suf, softmax_scale=1.0):
    desc = _suffix_desc(q_suf, k_suf, k_cache, ar_mask_suf, softmax_scale)
    return int(lib().pi_attn_suffix_workspace_bytes(ctypes.byref(desc)))


def pi_attn_suffix(q_suf, k_suf, v_suf, k_cache, v_cache, ar_mask_suf, out=None,
                   workspace=None, softmax_scale=1.0, stream=None, segment_ids=None,
                   cache_valid=None):
    """Suffix-only pass.  q_suf [B,Sq,Hq,d]; k_suf, v_suf [B,Sq,Hkv,d];
    k_cache, v_cache [B,P,Hkv,d]; ar_mask_suf uint8 [Sq] or [B,Sq].
    ``workspace``: a CUDA uint8 tensor of at least pi_attn_suffix_workspace_bytes
    (allocated here if None and needed).  ``segment_ids`` (int32, same layout
    as ar_mask_suf; negative = padding) and ``cache_valid`` (uint8 [B,P],
    nonzero = valid) select pi_attn_suffix_masked."""
    _need(q_suf, "q_suf", dims=4)
    _need(k_suf, "k_suf", q_suf.dtype, 4)
    _need(v_suf, "v_suf", q_suf.dtype, 4)
    _need(ar_mask_suf, "ar_mask_suf", torch.uint8)
    if k_cache is not None:
        _need(k_cache, "k_cache", q_suf.dtype, 4)
        _need(v_cache, "v_cache", q_suf.dtype, 4)
        if k_cache.shape != v_cache.shape or k_cache.shape[0] != q_suf.shape[0]:
            raise ValueError("cache shape mismatch")
    desc = _suffix_desc(q_suf, k_suf, k_cache, ar_mask_suf, softmax_scale)
    need = int(lib().pi_attn_suffix_workspace_bytes(ctypes.byref(desc)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_suf.device)
    if out is None:
        out = torch.empty_like(q_suf)
    _need(out, "out", q_suf.dtype, 4)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if segment_ids is None and cache_valid is None:
        rc = lib().pi_attn_suffix(ctypes.byref(desc), _ptr(q_suf), _ptr(k_suf), _ptr(v_suf),
                                  _ptr(k_cache), _ptr(v_cache), _ptr(ar_mask_suf), _ptr(out),
                                  _ptr(workspace), ws_bytes, ctypes.c_void_p(_stream(stream)))
        if rc != PI_OK:
            raise PiAttnError(rc, "pi_attn_suffix")
        return out
    if segment_ids is not None:
        _need(segment_ids, "segment_ids", torch.int32)
        if segment_ids.shape != ar_mask_suf.shape:
            raise ValueError("segment_ids must have the layout of ar_mask_suf")
    if cache_valid is not None:
        _need(cache_valid, "cache_valid", torch.uint8)
        if k_cache is None or tuple(cache_valid.shape) != tuple(k_cache.shape[:2]):
            raise ValueError("cache_valid must be [B, P]")
    rc = lib().pi_attn_suffix_masked(ctypes.byref(desc), _ptr(q_suf), _ptr(k_suf), _ptr(v_suf),
                                     _ptr(k_cache), _ptr(v_cache), _ptr(ar_mask_suf),
                                     _ptr(segment_ids), _ptr(cache_valid), _ptr(out),
                                     _ptr(workspace), ws_bytes, ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        raise PiAttnError(rc, "pi_attn_suffix_masked")
    return out


def pi_attn_suffix_noalloc(q_suf, k_suf, v_suf, k_cache, v_cache, ar_mask_suf, out,
                           softmax_scale=1.0, stream=None):
    """pi_attn_suffix with the split-K scratch in the library's fixed device
    buffer: allocates nothing, so ``out`` must be given."""
    _need(q_suf, "q_suf", dims=4)
    _need(k_suf, "k_suf", q_suf.dtype, 4)
    _need(v_suf, "v_suf", q_suf.dtype, 4)
    _need(ar_mask_suf, "ar_mask_suf", torch.uint8)
    if k_cache is not None:
        _need(k_cache, "k_cache", q_suf.dtype, 4)
        _need(v_cache, "v_cache", q_suf.dtype, 4)
        if k_cache.shape != v_cache.shape or k_cache.shape[0] != q_suf.shape[0]:
            raise ValueError("cache shape mismatch")
    _need(out, "out", q_suf.dtype, 4)
    desc = _suffix_desc(q_suf, k_suf, k_cache, ar_mask_suf, softmax_scale)
    rc = lib().pi_attn_suffix_noalloc(ctypes.byref(desc), _ptr(q_suf), _ptr(k_suf),
                                      _ptr(v_suf), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(ar_mask_suf), _ptr(out),
                                      ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        need = int(lib().pi_attn_suffix_workspace_bytes(ctypes.byref(desc)))
        cap = int(lib().pi_attn_suffix_noalloc_capacity())
        extra = (f": needs {need} bytes of scratch, the fixed buffer holds {cap}"
                 if rc == PI_ERR_UNSUPPORTED and need > cap else "")
        raise PiAttnError(rc, "pi_attn_suffix_noalloc" + extra)
    return out


def pi_rope_inplace(q, k, token_mask, prefix_mask=None, base=10000.0, positions=False,
                    stream=None):
    """Rotary embedding of q [B,S,Hq,d] (and k [B,S,Hkv,d] or None) in place at
    positions cumsum(token_mask) - 1 (+ the valid prefix count when
    ``prefix_mask`` [B,P] is given).  Returns the int32 [B,S] positions when
    ``positions`` is true."""
    _need(q, "q", dims=4)
    if k is not None:
        _need(k, "k", q.dtype, 4)
    _need(token_mask, "token_mask", torch.uint8)
    B, S, Hq, d = q.shape
    tbs = _mask_stride(token_mask, B, S)
    P, pbs = 0, 0
    if prefix_mask is not None:
        _need(prefix_mask, "prefix_mask", torch.uint8)
        P = prefix_mask.shape[-1]
        pbs = _mask_stride(prefix_mask, B, P)
    pos = torch.empty((B, S), dtype=torch.int32, device=q.device) if positions else None
    desc = PiRopeDesc(B, S, P, Hq, 1 if k is None else k.shape[2], d, _dtype_code(q),
                      float(base), tbs, pbs)
    rc = lib().pi_rope_inplace(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(token_mask),
                               _ptr(prefix_mask), _ptr(pos), ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        raise PiAttnError(rc, "pi_rope_inplace")
    return pos


def pi_euler_update(x, v, dt, stream=None):
    """x (fp32) += dt * v (bf16 or fp32, same number of elements), in place."""
    _need(x, "x", torch.float32)
    _need(v, "v")
    if v.numel() != x.numel():
        raise ValueError("x and v must have the same number of elements")
    rc = lib().pi_euler_update(_ptr(x), _ptr(v), _dtype_code(v), float(dt), x.numel(),
                               ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        raise PiAttnError(rc, "pi_euler_update")
    return x


def pi_attn_debug_mask(ar_mask, segment_ids=None, B=None, P=0, mode=0, stream=None):
    """The kernels' visibility matrix as uint8: [B,S,S] (mode 0) or [B,Sq,P+Sq] (mode 1)."""
    _need(ar_mask, "ar_mask", torch.uint8)
    S = ar_mask.shape[-1]
    if B is None:
        B = ar_mask.shape[0] if ar_mask.dim() == 2 else 1
    mbs = _mask_stride(ar_mask, B, S)
    if segment_ids is not None:
        _need(segment_ids, "segment_ids", torch.int32)
    Sk = S if mode == 0 else P + S
    out = torch.empty((B, S, Sk), dtype=torch.uint8, device=ar_mask.device)
    desc = PiAttnDesc(B, S, P if mode == 1 else 0, 1, 1, 256, PI_BF16, 1.0, mbs)
    rc = lib().pi_attn_debug_mask(ctypes.byref(desc), mode, _ptr(ar_mask), _ptr(segment_ids),
                                  _ptr(out), ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        raise PiAttnError(rc, "pi_attn_debug_mask")
    return out


def pi_attn_debug_tiles(ar_mask, segment_ids=None, B=None, Hq=8, stream=None):
    """The bf16 prefill kernel's tile classes: uint8 [B, ceil(S*Hq/256),
    ceil(S/128)], 0 = skipped, 1 = full, 2 = partial."""
    _need(ar_mask, "ar_mask", torch.uint8)
    S = ar_mask.shape[-1]
    if B is None:
        B = ar_mask.shape[0] if ar_mask.dim() == 2 else 1
    mbs = _mask_stride(ar_mask, B, S)
    if segment_ids is not None:
        _need(segment_ids, "segment_ids", torch.int32)
    n_pairs = (S * Hq + 255) // 256
    out = torch.empty((B, n_pairs, (S + 127) // 128), dtype=torch.uint8, device=ar_mask.device)
    desc = PiAttnDesc(B, S, 0, Hq, 1, 256, PI_BF16, 1.0, mbs)
    rc = lib().pi_attn_debug_tiles(ctypes.byref(desc), _ptr(ar_mask), _ptr(segment_ids),
                                   _ptr(out), ctypes.c_void_p(_stream(stream)))
    if rc != PI_OK:
        raise PiAttnError(rc, "pi_attn_debug_tiles")
    return out


def pi_attn_read_status(stream=None) -> int:
    return int(lib().pi_attn_read_status(ctypes.c_void_p(_stream(stream))))


def pi_attn_set_wait_limit(cycles: int) -> int:
    return int(lib().pi_attn_set_wait_limit(int(cycles)))


def pi_attn_selftest_wait(stream=None) -> int:
    return int(lib().pi_attn_selftest_wait(ctypes.c_void_p(_stream(stream))))
