"""Python binding of the C ABI in ``include/hsa.h`` (libhsa_b200.so).

Argument marshalling only: tensors are checked for device, dtype, shape and contiguity, outputs
and the workspace are allocated with torch on the input's device, and the C entry point of the same
name is called on the current torch stream. Every step of HSA runs in the CUDA library; there is
no fallback. If the library is missing or cannot be loaded, the first call raises.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhsa_b200.so")

HSA_OK = 0
STATUS_NAMES = {0: "HSA_OK", -1: "HSA_ERR_INVALID_ARG", -2: "HSA_ERR_UNSUPPORTED", -3: "HSA_ERR_WORKSPACE",
                -4: "HSA_ERR_CUDA", -5: "HSA_ERR_TIMEOUT"}

# C entry points and their argument types, as declared in include/hsa.h
_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_U = ctypes.c_uint
HSA_QK_NORM = 1
SIGNATURES = {
    "hsa_last_error": ([], ctypes.c_char_p),
    "hsa_workspace_status": ([_P, _P], _I),
    "hsa_forward_workspace_size": ([_I, _I, _I, _I, _I, _I], _SZ),
    "hsa_forward": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _SZ, _P], _I),
    "hsa_decode_workspace_size": ([_I, _I, _I64, _I, _I, _I], _SZ),
    "hsa_decode": ([_P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _SZ, _P], _I),
    "hsa_decode_noalloc": ([_P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P], _I),
    "hsa_backward_workspace_size": ([_I, _I, _I, _I, _I, _I], _SZ),
    "hsa_backward": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _SZ, _P],
                     _I),
    "hsa_forward_ex_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _U], _SZ),
    "hsa_forward_ex": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _U, _P, _P, _P, _P, _SZ, _P], _I),
    "hsa_decode_ex_workspace_size": ([_I, _I, _I, _I, _I64, _I, _I, _I, _U], _SZ),
    "hsa_decode_ex": ([_P, _P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _F, _U, _P, _P, _P, _P, _SZ, _P],
                      _I),
    "hsa_backward_ex_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _U], _SZ),
    "hsa_backward_ex": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _U, _P, _P, _P, _P, _P,
                         _P, _SZ, _P], _I),
    "hsa_forward_varlen_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _U], _SZ),
    "hsa_forward_varlen": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _U, _P, _P, _P, _P, _SZ, _P],
                           _I),
    "hsa_backward_varlen_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _U], _SZ),
    "hsa_backward_varlen": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _U, _P, _P,
                             _P, _P, _P, _P, _SZ, _P], _I),
    "hsa_selftest_bounded_wait": ([_P, _SZ, _U, _P], _I),
    "hsa_profile_enable": ([_I], _I),
    "hsa_profile_summary": ([ctypes.c_char_p, _SZ], _I),
}

_lib = None


class HSAError(RuntimeError):
    def __init__(self, name, status, message):
        super().__init__(f"{name} failed: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def lib():
    """Load libhsa_b200.so (once) and declare its entry points. Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with ultra_long_context_b200/build.py "
                               "(or __graft_entry__.build()); there is no fallback path")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def hsa_last_error():
    return lib().hsa_last_error().decode()


def _check(name, status):
    if status != HSA_OK:
        raise HSAError(name, status, hsa_last_error())


def hsa_workspace_status(workspace, stream=None):
    """Device-side status of the last call that used ``workspace`` (a uint8 CUDA tensor): synchronizes
    the stream and raises HSAError (HSA_ERR_TIMEOUT) if a bounded device wait of that call ran out."""
    if not (isinstance(workspace, torch.Tensor) and workspace.is_cuda):
        raise ValueError("workspace must be a CUDA tensor")
    _check("hsa_workspace_status", lib().hsa_workspace_status(_ptr(workspace), _stream(workspace.device, stream)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, shape, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return None
    if workspace is not None:
        return workspace
    # +256 so a 256-byte aligned window always fits
    return torch.empty(nbytes + 256, dtype=torch.uint8, device=device)


def _aligned(ws):
    if ws is None:
        return None, 0
    p = ws.data_ptr()
    off = (-p) % 256
    return ctypes.c_void_p(p + off), ws.numel() * ws.element_size() - off


def hsa_forward_workspace_size(B, H, T, D, chunk=64, topk=16):
    return int(lib().hsa_forward_workspace_size(B, H, T, D, chunk, topk))


def hsa_forward_ex_workspace_size(B, H, Hkv, T, D, chunk=64, topk=16, flags=0):
    return int(lib().hsa_forward_ex_workspace_size(B, H, Hkv, T, D, chunk, topk, flags))


def _flags(qk_norm):
    return HSA_QK_NORM if qk_norm else 0


def hsa_forward(Q, K, V, L, topk, scale=0.0, chunk=64, out=None, sel_idx=None, sel_w=None, workspace=None,
                stream=None, return_selection=True, Qs=None, qk_norm=False):
    """HSA prefill forward. Q [B, H, T, D], K, V [B, Hkv, T, D], L [B, Hkv, T // 64, D] bf16 (CUDA); Hkv = H
    unless key/value heads are grouped (query head h uses head h // (H // Hkv)).

    Qs: separate retrieval queries [B, H, T, D] bf16 (Qs scores the landmarks, Q attends), or None when Q
    does both. qk_norm: Step 3 attends with the L2-normalised query and keys. Any of the three calls
    hsa_forward_ex, else hsa_forward.
    Returns (out [B, H, T, D] bf16, sel_idx [B, H, T, topk] int32, sel_w [B, H, T, topk] fp32); the
    selection is None when ``return_selection`` is False and none was passed in.
    """
    B, H, T, D = Q.shape
    Hkv = K.shape[1]
    dev = Q.device
    _need(Q, "Q", torch.bfloat16, (B, H, T, D), dev)
    if Qs is not None:
        _need(Qs, "Qs", torch.bfloat16, (B, H, T, D), dev)
    for n, t in (("K", K), ("V", V)):
        _need(t, n, torch.bfloat16, (B, Hkv, T, D), dev)
    _need(L, "L", torch.bfloat16, (B, Hkv, T // chunk, D), dev)
    if out is None:
        out = torch.empty_like(Q)
    _need(out, "out", torch.bfloat16, (B, H, T, D), dev)
    if return_selection and sel_idx is None:
        sel_idx = torch.empty((B, H, T, topk), dtype=torch.int32, device=dev)
    if return_selection and sel_w is None:
        sel_w = torch.empty((B, H, T, topk), dtype=torch.float32, device=dev)
    if Qs is None and not qk_norm and Hkv == H:
        nbytes = hsa_forward_workspace_size(B, H, T, D, chunk, topk)
        ws = _workspace(nbytes, dev, workspace)
        wp, wn = _aligned(ws)
        st = lib().hsa_forward(_ptr(Q), _ptr(K), _ptr(V), _ptr(L), B, H, T, D, chunk, topk, float(scale), _ptr(out),
                               _ptr(sel_idx), _ptr(sel_w), wp, wn, _stream(dev, stream))
        _check("hsa_forward", st)
    else:
        fl = _flags(qk_norm)
        ws = _workspace(hsa_forward_ex_workspace_size(B, H, Hkv, T, D, chunk, topk, fl), dev, workspace)
        wp, wn = _aligned(ws)
        st = lib().hsa_forward_ex(_ptr(Qs), _ptr(Q), _ptr(K), _ptr(V), _ptr(L), B, H, Hkv, T, D, chunk, topk,
                                  float(scale), fl, _ptr(out), _ptr(sel_idx), _ptr(sel_w), wp, wn,
                                  _stream(dev, stream))
        _check("hsa_forward_ex", st)
    return out, sel_idx, sel_w


def hsa_decode_workspace_size(B, H, Tmax, D, chunk=64, topk=16):
    return int(lib().hsa_decode_workspace_size(B, H, Tmax, D, chunk, topk))


def hsa_decode_ex_workspace_size(B, H, Hkv, Tmax, D, chunk=64, topk=16, flags=0, Tq=1):
    return int(lib().hsa_decode_ex_workspace_size(B, H, Hkv, Tq, Tmax, D, chunk, topk, flags))


def hsa_decode(q, Kc, Vc, Lc, cache_len, topk, scale=0.0, chunk=64, out=None, sel_idx=None, sel_w=None,
               workspace=None, stream=None, qs=None, qk_norm=False):
    """HSA decode. q [B, H, D] (or [B, H, Tq, D]: the last Tq tokens of each cache in one step),
    Kc / Vc [B, Hkv, Tmax, D], Lc [B, Hkv, Tmax // 64, D] bf16; cache_len [B] int64 (Hkv = H unless key/value
    heads are grouped).

    qs: a separate retrieval query shaped like q, or None when q does both. qk_norm: Step 3 attends with
    the L2-normalised query and keys. Any option (or Tq > 1) calls hsa_decode_ex, else hsa_decode.
    Returns (out shaped like q, sel_idx [..., topk] int32, sel_w [..., topk] fp32).
    """
    multi = q.dim() == 4
    B, H, D = q.shape[0], q.shape[1], q.shape[-1]
    Tq = q.shape[2] if multi else 1
    qshape = tuple(q.shape)
    Hkv, Tmax = Kc.shape[1], Kc.shape[2]
    dev = q.device
    _need(q, "q", torch.bfloat16, qshape, dev)
    if qs is not None:
        _need(qs, "qs", torch.bfloat16, qshape, dev)
    _need(Kc, "Kc", torch.bfloat16, (B, Hkv, Tmax, D), dev)
    _need(Vc, "Vc", torch.bfloat16, (B, Hkv, Tmax, D), dev)
    _need(Lc, "Lc", torch.bfloat16, (B, Hkv, Tmax // chunk, D), dev)
    _need(cache_len, "cache_len", torch.int64, (B,), dev)
    if out is None:
        out = torch.empty_like(q)
    if sel_idx is None:
        sel_idx = torch.empty(qshape[:-1] + (topk,), dtype=torch.int32, device=dev)
    if sel_w is None:
        sel_w = torch.empty(qshape[:-1] + (topk,), dtype=torch.float32, device=dev)
    if qs is None and not qk_norm and Hkv == H and not multi:
        nbytes = hsa_decode_workspace_size(B, H, Tmax, D, chunk, topk)
        ws = _workspace(nbytes, dev, workspace)
        wp, wn = _aligned(ws)
        st = lib().hsa_decode(_ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Lc), _ptr(cache_len), Tmax, B, H, D, chunk, topk,
                              float(scale), _ptr(out), _ptr(sel_idx), _ptr(sel_w), wp, wn, _stream(dev, stream))
        _check("hsa_decode", st)
    else:
        fl = _flags(qk_norm)
        ws = _workspace(hsa_decode_ex_workspace_size(B, H, Hkv, Tmax, D, chunk, topk, fl, Tq), dev, workspace)
        wp, wn = _aligned(ws)
        st = lib().hsa_decode_ex(_ptr(qs), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Lc), _ptr(cache_len), Tmax, B, H, Hkv,
                                 Tq, D, chunk, topk, float(scale), fl, _ptr(out), _ptr(sel_idx), _ptr(sel_w), wp, wn,
                                 _stream(dev, stream))
        _check("hsa_decode_ex", st)
    return out, sel_idx, sel_w


def hsa_decode_noalloc(q, Kc, Vc, Lc, cache_len, topk, scale=0.0, chunk=64, out=None, sel_idx=None, sel_w=None,
                       stream=None):
    """HSA decode with no allocation inside the call: the library's fixed scratch array replaces the
    workspace (for callers that cannot allocate device memory while they decode). Same arguments and
    results as hsa_decode. Calls share that array, so calls overlapping on the GPU race; the first
    call on a device sets up the array's address and should come before any stream capture."""
    B, H, D = q.shape
    Tmax = Kc.shape[2]
    dev = q.device
    _need(q, "q", torch.bfloat16, (B, H, D), dev)
    _need(Kc, "Kc", torch.bfloat16, (B, H, Tmax, D), dev)
    _need(Vc, "Vc", torch.bfloat16, (B, H, Tmax, D), dev)
    _need(Lc, "Lc", torch.bfloat16, (B, H, Tmax // chunk, D), dev)
    _need(cache_len, "cache_len", torch.int64, (B,), dev)
    if out is None:
        out = torch.empty_like(q)
    if sel_idx is None:
        sel_idx = torch.empty((B, H, topk), dtype=torch.int32, device=dev)
    if sel_w is None:
        sel_w = torch.empty((B, H, topk), dtype=torch.float32, device=dev)
    st = lib().hsa_decode_noalloc(_ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Lc), _ptr(cache_len), Tmax, B, H, D, chunk, topk,
                                  float(scale), _ptr(out), _ptr(sel_idx), _ptr(sel_w), _stream(dev, stream))
    _check("hsa_decode_noalloc", st)
    return out, sel_idx, sel_w


def hsa_backward_workspace_size(B, H, T, D, chunk=64, topk=16):
    return int(lib().hsa_backward_workspace_size(B, H, T, D, chunk, topk))


def hsa_backward_ex_workspace_size(B, H, Hkv, T, D, chunk=64, topk=16, flags=0):
    return int(lib().hsa_backward_ex_workspace_size(B, H, Hkv, T, D, chunk, topk, flags))


def hsa_backward(Q, K, V, L, out, dout, sel_idx, sel_w, scale=0.0, chunk=64, grads=None, workspace=None,
                 stream=None, Qs=None, qk_norm=False):
    """Backward of hsa_forward for its selection (same options). Returns (dQ, dK, dV, dL), fp32, shaped like
    Q, K, V, L; with separate retrieval queries Qs, (dQ, dK, dV, dL, dQs) where dQ is the attention
    query's gradient. Any option (Qs, qk_norm, grouped heads) calls hsa_backward_ex."""
    B, H, T, D = Q.shape
    Hkv = K.shape[1]
    topk = sel_idx.shape[-1]
    dev = Q.device
    if Qs is not None:
        _need(Qs, "Qs", torch.bfloat16, (B, H, T, D), dev)
    for n, t in (("Q", Q), ("out", out), ("dout", dout)):
        _need(t, n, torch.bfloat16, (B, H, T, D), dev)
    for n, t in (("K", K), ("V", V)):
        _need(t, n, torch.bfloat16, (B, Hkv, T, D), dev)
    _need(L, "L", torch.bfloat16, (B, Hkv, T // chunk, D), dev)
    _need(sel_idx, "sel_idx", torch.int32, (B, H, T, topk), dev)
    _need(sel_w, "sel_w", torch.float32, (B, H, T, topk), dev)
    if grads is None:
        grads = (torch.empty((B, H, T, D), dtype=torch.float32, device=dev),
                 torch.empty((B, Hkv, T, D), dtype=torch.float32, device=dev),
                 torch.empty((B, Hkv, T, D), dtype=torch.float32, device=dev),
                 torch.empty((B, Hkv, T // chunk, D), dtype=torch.float32, device=dev))
    dQ, dK, dV, dL = grads[:4]
    if Qs is None and not qk_norm and Hkv == H:
        nbytes = hsa_backward_workspace_size(B, H, T, D, chunk, topk)
        ws = _workspace(nbytes, dev, workspace)
        wp, wn = _aligned(ws)
        st = lib().hsa_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(L), _ptr(out), _ptr(dout), _ptr(sel_idx),
                                _ptr(sel_w), B, H, T, D, chunk, topk, float(scale), _ptr(dQ), _ptr(dK), _ptr(dV),
                                _ptr(dL) if dL.numel() else None, wp, wn, _stream(dev, stream))
        _check("hsa_backward", st)
        return dQ, dK, dV, dL
    dQs = None
    if Qs is not None:
        dQs = grads[4] if len(grads) > 4 else torch.empty((B, H, T, D), dtype=torch.float32, device=dev)
    fl = _flags(qk_norm)
    ws = _workspace(hsa_backward_ex_workspace_size(B, H, Hkv, T, D, chunk, topk, fl), dev, workspace)
    wp, wn = _aligned(ws)
    st = lib().hsa_backward_ex(_ptr(Qs), _ptr(Q), _ptr(K), _ptr(V), _ptr(L), _ptr(out), _ptr(dout), _ptr(sel_idx),
                               _ptr(sel_w), B, H, Hkv, T, D, chunk, topk, float(scale), fl, _ptr(dQ), _ptr(dK),
                               _ptr(dV), _ptr(dL) if dL.numel() else None, _ptr(dQs), wp, wn, _stream(dev, stream))
    _check("hsa_backward_ex", st)
    return (dQ, dK, dV, dL) if Qs is None else (dQ, dK, dV, dL, dQs)


def _varlen_shapes(Q, K, L, cu_seqlens, chunk):
    total, H, D = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or B < 1:
        raise ValueError("cu_seqlens must be an int32 CUDA tensor of B + 1 offsets")
    return total, H, Hkv, D, B


def hsa_forward_varlen(Q, K, V, L, cu_seqlens, max_seqlen, topk, scale=0.0, chunk=64, out=None, sel_idx=None,
                       sel_w=None, workspace=None, stream=None, Qs=None, qk_norm=False):
    """HSA forward of a variable-length batch in the packed token-major layout: Q [total, H, D], K, V
    [total, Hkv, D], L [total_chunks, Hkv, D] bf16 (each sequence's floor(len / 64) landmarks in order),
    cu_seqlens [B + 1] int32 on the device, every length <= max_seqlen. Returns (out [total, H, D],
    sel_idx / sel_w [total, H, topk]; chunk ids within each sequence)."""
    total, H, Hkv, D, B = _varlen_shapes(Q, K, L, cu_seqlens, chunk)
    dev = Q.device
    _need(Q, "Q", torch.bfloat16, (total, H, D), dev)
    if Qs is not None:
        _need(Qs, "Qs", torch.bfloat16, (total, H, D), dev)
    for n, t in (("K", K), ("V", V)):
        _need(t, n, torch.bfloat16, (total, Hkv, D), dev)
    _need(L, "L", torch.bfloat16, (L.shape[0], Hkv, D), dev)
    out = torch.empty_like(Q) if out is None else out
    sel_idx = torch.empty((total, H, topk), dtype=torch.int32, device=dev) if sel_idx is None else sel_idx
    sel_w = torch.empty((total, H, topk), dtype=torch.float32, device=dev) if sel_w is None else sel_w
    fl = _flags(qk_norm)
    ws = _workspace(int(lib().hsa_forward_varlen_workspace_size(B, H, Hkv, max_seqlen, D, chunk, topk, fl)), dev,
                    workspace)
    wp, wn = _aligned(ws)
    st = lib().hsa_forward_varlen(_ptr(Qs), _ptr(Q), _ptr(K), _ptr(V), _ptr(L) if L.numel() else _ptr(Q),
                                  _ptr(cu_seqlens), B, max_seqlen, H, Hkv, D, chunk, topk, float(scale), fl, _ptr(out),
                                  _ptr(sel_idx), _ptr(sel_w), wp, wn, _stream(dev, stream))
    _check("hsa_forward_varlen", st)
    return out, sel_idx, sel_w


def hsa_backward_varlen(Q, K, V, L, out, dout, sel_idx, sel_w, cu_seqlens, max_seqlen, scale=0.0, chunk=64,
                        workspace=None, stream=None, Qs=None, qk_norm=False):
    """Backward of hsa_forward_varlen for its selection. Returns (dQ, dK, dV, dL) fp32 in the packed
    layout (and dQs with a separate retrieval query)."""
    total, H, Hkv, D, B = _varlen_shapes(Q, K, L, cu_seqlens, chunk)
    topk = sel_idx.shape[-1]
    dev = Q.device
    for n, t in (("Q", Q), ("out", out), ("dout", dout)):
        _need(t, n, torch.bfloat16, (total, H, D), dev)
    for n, t in (("K", K), ("V", V)):
        _need(t, n, torch.bfloat16, (total, Hkv, D), dev)
    _need(sel_idx, "sel_idx", torch.int32, (total, H, topk), dev)
    _need(sel_w, "sel_w", torch.float32, (total, H, topk), dev)
    dQ = torch.empty((total, H, D), dtype=torch.float32, device=dev)
    dK = torch.empty((total, Hkv, D), dtype=torch.float32, device=dev)
    dV = torch.empty((total, Hkv, D), dtype=torch.float32, device=dev)
    dL = torch.empty(tuple(L.shape), dtype=torch.float32, device=dev)
    dQs = torch.empty_like(dQ) if Qs is not None else None
    fl = _flags(qk_norm)
    ws = _workspace(int(lib().hsa_backward_varlen_workspace_size(B, H, Hkv, max_seqlen, D, chunk, topk, fl)), dev,
                    workspace)
    wp, wn = _aligned(ws)
    # a zero-row L / dL still needs a valid (never read) 16-byte aligned pointer
    lp = _ptr(L) if L.numel() else _ptr(Q)
    dlp = _ptr(dL) if dL.numel() else _ptr(dQ)
    st = lib().hsa_backward_varlen(_ptr(Qs), _ptr(Q), _ptr(K), _ptr(V), lp, _ptr(out), _ptr(dout), _ptr(sel_idx),
                                   _ptr(sel_w), _ptr(cu_seqlens), B, max_seqlen, H, Hkv, D, chunk, topk, float(scale),
                                   fl, _ptr(dQ), _ptr(dK), _ptr(dV), dlp, _ptr(dQs), wp, wn, _stream(dev, stream))
    _check("hsa_backward_varlen", st)
    return (dQ, dK, dV, dL) if Qs is None else (dQ, dK, dV, dL, dQs)


def hsa_profile_enable(on=True):
    lib().hsa_profile_enable(1 if on else 0)


def hsa_profile_summary():
    """{launch site: (launches, total device ms)} for the launches recorded since profiling was enabled."""
    n = lib().hsa_profile_summary(None, 0)
    if n < 0:
        raise RuntimeError("hsa_profile_summary failed")
    buf = ctypes.create_string_buffer(n + 1)
    lib().hsa_profile_summary(buf, n + 1)
    res = {}
    for line in buf.value.decode().splitlines():
        name, cnt, ms = line.split(",")
        res[name] = (int(cnt), float(ms))
    return res


def default_scale(D):
    return 1.0 / math.sqrt(D)
