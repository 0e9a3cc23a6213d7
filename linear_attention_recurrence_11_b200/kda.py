"""Python binding of libkda.so (declared in include/kda.h).

Argument marshalling only: torch tensors (CUDA, contiguous) are checked for
shape/dtype and passed to the C ABI as raw device pointers with the current
(or given) CUDA stream; every step of the computation runs in the library's
kernels. Output tensors are allocated here with torch when the caller does not
pass them. There is no CPU fallback: importing this module raises if
``libkda.so`` has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libkda.so is not built ({LIB_PATH}); run "
                      "`python -m linear_attention_recurrence_11_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.kda_status_string.argtypes = [_i]
_lib.kda_status_string.restype = ctypes.c_char_p
_lib.kda_abi_version.restype = _i
_lib.kda_last_cuda_error.restype = ctypes.c_char_p
_lib.kda_forward_workspace_size.argtypes = [_i] * 8
_lib.kda_forward_workspace_size.restype = _sz
_lib.kda_forward_workspace_size_ex.argtypes = [_i] * 9
_lib.kda_forward_workspace_size_ex.restype = _sz
_lib.kda_forward_launches.argtypes = [_i] * 10
_lib.kda_forward_launches.restype = _i
_FWD = [_vp] * 8 + [_i] * 7 + [_vp, _i, _vp, _sz, _vp, _vp]
_lib.kda_forward.argtypes = _FWD
_lib.kda_forward.restype = _i
_lib.kda_forward_ex.argtypes = _FWD + [_i]
_lib.kda_forward_ex.restype = _i
_lib.kda_decode_step.argtypes = [_vp] * 7 + [_i] * 5 + [_vp]
_lib.kda_decode_step.restype = _i
_lib.kda_forward_noalloc.argtypes = [_vp] * 8 + [_i] * 7 + [_vp, _i, _vp, _vp]
_lib.kda_forward_noalloc.restype = _i
_lib.kda_forward_segmented_workspace_size.argtypes = [_i] * 8
_lib.kda_forward_segmented_workspace_size.restype = _sz
_lib.kda_forward_segmented_launches.argtypes = [_i] * 9
_lib.kda_forward_segmented_launches.restype = _i
_lib.kda_forward_segmented.argtypes = [_vp] * 8 + [_i] * 8 + [_vp, _sz, _vp, _vp, _i]
_lib.kda_forward_segmented.restype = _i
_lib.kda_forward_segmented_varlen_workspace_size.argtypes = [_i] * 8
_lib.kda_forward_segmented_varlen_workspace_size.restype = _sz
_lib.kda_forward_segmented_varlen_launches.argtypes = [_i] * 9
_lib.kda_forward_segmented_varlen_launches.restype = _i
_lib.kda_forward_segmented_varlen.argtypes = [_vp] * 8 + [_i] * 6 + [_vp, _i, _i, _vp, _sz, _vp, _vp, _i]
_lib.kda_forward_segmented_varlen.restype = _i
_lib.kda_decode_multi.argtypes = [_vp] * 8 + [_i] * 6 + [_vp, _vp]
_lib.kda_decode_multi.restype = _i
_lib.kda_forward_snapshots.argtypes = [_vp] * 9 + [_i] * 8 + [_vp, _sz, _vp, _vp, _i]
_lib.kda_forward_snapshots.restype = _i
_lib.kda_segment_pair.argtypes = [_vp] * 7 + [_i] * 7 + [_vp, _vp, _i]
_lib.kda_segment_pair.restype = _i
_lib.kda_kcp_scan.argtypes = [_vp] * 5 + [_i] * 5 + [_vp]
_lib.kda_kcp_scan.restype = _i
_lib.kda_selftest_wait_timeout.argtypes = [_vp, ctypes.c_longlong, _vp]
_lib.kda_selftest_wait_timeout.restype = _i
_lib.kda_forward_fused.argtypes = _FWD + [_i, _i]
_lib.kda_forward_fused.restype = _i
_lib.kda_decode_step_fused.argtypes = [_vp] * 7 + [_i] * 5 + [_vp, _i]
_lib.kda_decode_step_fused.restype = _i
_lib.kda_forward_host_workspace_size.argtypes = [_i] * 8
_lib.kda_forward_host_workspace_size.restype = _sz
_lib.kda_forward_host.argtypes = [_vp] * 8 + [_i] * 8 + [_vp, _sz, _vp, _vp, _i]
_lib.kda_forward_host.restype = _i
_lib.kda_forward_host_varlen_workspace_size.argtypes = [_i] * 6 + [_vp, _i, _i]
_lib.kda_forward_host_varlen_workspace_size.restype = _sz
_lib.kda_forward_host_varlen.argtypes = [_vp] * 8 + [_i] * 6 + [_vp, _i, _i, _vp, _sz, _vp, _vp, _i]
_lib.kda_forward_host_varlen.restype = _i

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_ALIGNMENT = 0, 1, 2, 3
KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_ERR_SCRATCH_LIMIT = 4, 5, 6, 7
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
PATHS = {"auto": 0, "simt": 1, "tc": 2, "tc_single": 3, "tc_split": 4, "tc_pipe": 5}
KDA_FUSE_NORM_QK, KDA_FUSE_GATE_LOGITS = 1, 2  # fused pre-operations (see include/kda.h)


class KdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = f": {_lib.kda_last_cuda_error().decode()}" if code == KDA_ERR_CUDA else ""
        super().__init__(f"{where}: {kda_status_string(code)}{detail} (status {code})")


def kda_status_string(code: int) -> str:
    return _lib.kda_status_string(int(code)).decode()


def kda_abi_version() -> int:
    return _lib.kda_abi_version()


def kda_forward_workspace_size(B, T, H, dk, dv, chunk, num_seqs, dtype, path="auto") -> int:
    n = _lib.kda_forward_workspace_size_ex(B, T, H, dk, dv, chunk, num_seqs, DTYPES.get(dtype, dtype), PATHS[path])
    if n == ctypes.c_size_t(-1).value:
        raise KdaError(KDA_ERR_UNSUPPORTED if path.startswith("tc") else KDA_ERR_INVALID_ARG,
                       "kda_forward_workspace_size")
    return int(n)


def kda_forward_launches(B, T, H, dk, dv, chunk, dtype, has_cu_seqlens, num_seqs, path="auto") -> int:
    return _lib.kda_forward_launches(B, T, H, dk, dv, chunk, DTYPES.get(dtype, dtype),
                                     int(bool(has_cu_seqlens)), num_seqs, PATHS[path])


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def kda_forward(q, k, v, g, beta, S0=None, *, chunk: int = 64, cu_seqlens=None, o=None,
                S_T=None, return_state: bool = True, workspace=None, dev_status=None,
                stream=None, path: str = "auto", fuse: int = 0):
    """Chunked KDA prefill. q, k, g ``[B, T, H, dk]``; v ``[B, T, H, dv]``;
    beta ``[B, T, H]`` (fp32 or bf16, all the same); S0 ``[N, H, dv, dk]`` fp32
    or None; cu_seqlens int32 ``[N+1]`` (B must be 1) or None. ``fuse``:
    KDA_FUSE_* bits (raw q, k normalised in the kernel; g as gate logits).
    Returns ``(o, S_T)`` (S_T None when ``return_state`` is False)."""
    _need(k, "k")
    dtype, dev = k.dtype, k.device
    if dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {dtype}")
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    _need(q, "q", dtype, (B, T, H, dk), dev)
    _need(g, "g", dtype, (B, T, H, dk), dev)
    _need(v, "v", dtype, (B, T, H, dv), dev)
    _need(beta, "beta", dtype, (B, T, H), dev)
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if S0 is not None:
        _need(S0, "S0", torch.float32, (N, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dtype, device=dev)
    _need(o, "o", dtype, (B, T, H, dv), dev)
    if return_state and S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (N, H, dv, dk), dev)
    if workspace is None:
        ws_need = _lib.kda_forward_workspace_size_ex(B, T, H, dk, dv, int(chunk), N, DTYPES[dtype], PATHS[path])
        if ws_need not in (0, ctypes.c_size_t(-1).value):
            workspace = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv,
            int(chunk), DTYPES[dtype], _ptr(cu_seqlens), N if cu_seqlens is not None else 0,
            _ptr(workspace), ws_bytes, _ptr(dev_status), _stream_handle(stream, dev), PATHS[path])
    rc = _lib.kda_forward_fused(*args, int(fuse)) if fuse else _lib.kda_forward_ex(*args)
    if rc != KDA_OK:
        raise KdaError(rc, "kda_forward")
    return o, S_T


def kda_forward_noalloc(q, k, v, g, beta, S0, o, S_T, *, chunk: int = 64, cu_seqlens=None,
                        dev_status=None, stream=None):
    """kda_forward for callers that cannot allocate device memory: no workspace
    argument (the library keeps a fixed 8 KiB schedule array per device) and no
    allocation here either, so o and S_T must be passed in (S_T may be None).
    Packed batches are limited to 2048 sequences (KdaError KDA_ERR_SCRATCH_LIMIT
    beyond that). Calls that overlap on one device race on that array."""
    _need(k, "k")
    dtype, dev = k.dtype, k.device
    if dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {dtype}")
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    _need(q, "q", dtype, (B, T, H, dk), dev)
    _need(g, "g", dtype, (B, T, H, dk), dev)
    _need(v, "v", dtype, (B, T, H, dv), dev)
    _need(beta, "beta", dtype, (B, T, H), dev)
    N = B
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        N = cu_seqlens.numel() - 1
    if S0 is not None:
        _need(S0, "S0", torch.float32, (N, H, dv, dk), dev)
    _need(o, "o", dtype, (B, T, H, dv), dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (N, H, dv, dk), dev)
    with torch.cuda.device(dev):  # the library's scratch array is the current device's
        rc = _lib.kda_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                      _ptr(S_T), B, T, H, dk, dv, int(chunk), DTYPES[dtype],
                                      _ptr(cu_seqlens), N if cu_seqlens is not None else 0,
                                      _ptr(dev_status), _stream_handle(stream, dev))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_forward_noalloc")
    return o, S_T


def _need_host(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def kda_forward_host_workspace_size(B, T, H, dk, dv, chunk, dtype, piece_len=0) -> int:
    n = _lib.kda_forward_host_workspace_size(B, T, H, dk, dv, chunk, DTYPES.get(dtype, dtype), int(piece_len))
    if n == ctypes.c_size_t(-1).value:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_forward_host_workspace_size")
    return int(n)


def kda_forward_host_varlen_workspace_size(T, H, dk, dv, chunk, dtype, cu_seqlens, piece_len=0) -> int:
    cu = torch.as_tensor(cu_seqlens, dtype=torch.int32).contiguous()
    n = _lib.kda_forward_host_varlen_workspace_size(T, H, dk, dv, chunk, DTYPES.get(dtype, dtype), _ptr(cu),
                                                    cu.numel() - 1, int(piece_len))
    if n == ctypes.c_size_t(-1).value:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_forward_host_varlen_workspace_size")
    return int(n)


def kda_forward_host(q, k, v, g, beta, S0=None, *, chunk: int = 64, piece_len: int = 0, cu_seqlens=None, o=None,
                     S_T=None, return_state: bool = True, workspace=None, device=None, dev_status=None, stream=None,
                     path: str = "auto"):
    """Prefill with inputs and outputs in host memory (CPU tensors, pinned for
    overlapped copies): the library uploads, runs and downloads the tokens in
    pieces of about ``piece_len`` (0: about T / 8). Dense batches ``[B, T, H, d]``,
    or with ``cu_seqlens`` (a CPU int32 tensor ``[N + 1]``, B must be 1) a packed
    batch whose states are ``[N, H, dv, dk]``. Outputs are allocated on the host
    (pinned when k is) unless given. Returns ``(o, S_T)``; they are complete once
    ``stream`` (default: the current stream of ``device``) has finished."""
    if cu_seqlens is not None:
        return _forward_host_varlen(q, k, v, g, beta, S0, chunk=chunk, piece_len=piece_len, cu_seqlens=cu_seqlens,
                                    o=o, S_T=S_T, return_state=return_state, workspace=workspace, device=device,
                                    dev_status=dev_status, stream=stream, path=path)
    _need_host(k, "k")
    dtype = k.dtype
    if dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {dtype}")
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    _need_host(q, "q", dtype, (B, T, H, dk))
    _need_host(g, "g", dtype, (B, T, H, dk))
    _need_host(v, "v", dtype, (B, T, H, dv))
    _need_host(beta, "beta", dtype, (B, T, H))
    if S0 is not None:
        _need_host(S0, "S0", torch.float32, (B, H, dv, dk))
    pin = k.is_pinned()
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dtype, pin_memory=pin)
    _need_host(o, "o", dtype, (B, T, H, dv))
    if return_state and S_T is None:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, pin_memory=pin)
    if S_T is not None:
        _need_host(S_T, "S_T", torch.float32, (B, H, dv, dk))
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if workspace is None:
        workspace = torch.empty(kda_forward_host_workspace_size(B, T, H, dk, dv, chunk, dtype, piece_len),
                                dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, None, dev)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, None, dev)
    with torch.cuda.device(dev):
        rc = _lib.kda_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T),
                                   B, T, H, dk, dv, int(chunk), DTYPES[dtype], int(piece_len), _ptr(workspace),
                                   workspace.numel(), _ptr(dev_status), _stream_handle(stream, dev), PATHS[path])
    if rc != KDA_OK:
        raise KdaError(rc, "kda_forward_host")
    return o, S_T


def _forward_host_varlen(q, k, v, g, beta, S0, *, chunk, piece_len, cu_seqlens, o, S_T, return_state, workspace,
                         device, dev_status, stream, path):
    _need_host(k, "k")
    dtype = k.dtype
    if dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {dtype}")
    B, T, H, dk = k.shape
    if B != 1:
        raise ValueError("cu_seqlens needs B == 1")
    dv = v.shape[-1]
    _need_host(q, "q", dtype, (B, T, H, dk))
    _need_host(g, "g", dtype, (B, T, H, dk))
    _need_host(v, "v", dtype, (B, T, H, dv))
    _need_host(beta, "beta", dtype, (B, T, H))
    cu = cu_seqlens
    _need_host(cu, "cu_seqlens", torch.int32, None)
    N = cu.numel() - 1
    if S0 is not None:
        _need_host(S0, "S0", torch.float32, (N, H, dv, dk))
    pin = k.is_pinned()
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dtype, pin_memory=pin)
    _need_host(o, "o", dtype, (B, T, H, dv))
    if return_state and S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, pin_memory=pin)
    if S_T is not None:
        _need_host(S_T, "S_T", torch.float32, (N, H, dv, dk))
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if workspace is None:
        workspace = torch.empty(kda_forward_host_varlen_workspace_size(T, H, dk, dv, chunk, dtype, cu, piece_len),
                                dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, None, dev)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, None, dev)
    with torch.cuda.device(dev):
        rc = _lib.kda_forward_host_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                          _ptr(S_T), T, H, dk, dv, int(chunk), DTYPES[dtype], _ptr(cu), N,
                                          int(piece_len), _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                          _stream_handle(stream, dev), PATHS[path])
    if rc != KDA_OK:
        raise KdaError(rc, "kda_forward_host_varlen")
    return o, S_T


def kda_forward_segmented_workspace_size(B, T, H, dk, dv, chunk, dtype, seg_len) -> int:
    n = _lib.kda_forward_segmented_workspace_size(B, T, H, dk, dv, chunk, DTYPES.get(dtype, dtype), seg_len)
    if n == ctypes.c_size_t(-1).value:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_forward_segmented_workspace_size")
    return int(n)


def kda_forward_segmented_launches(B, T, H, dk, dv, chunk, dtype, seg_len, path="auto") -> int:
    return _lib.kda_forward_segmented_launches(B, T, H, dk, dv, chunk, DTYPES.get(dtype, dtype), seg_len,
                                               PATHS[path])


def kda_forward_segmented_varlen_workspace_size(T, H, dk, dv, chunk, dtype, num_seqs, seg_len) -> int:
    n = _lib.kda_forward_segmented_varlen_workspace_size(T, H, dk, dv, chunk, DTYPES.get(dtype, dtype), num_seqs,
                                                         seg_len)
    if n == ctypes.c_size_t(-1).value:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_forward_segmented_varlen_workspace_size")
    return int(n)


def kda_forward_segmented_varlen_launches(T, H, dk, dv, chunk, dtype, num_seqs, seg_len, path="auto") -> int:
    return _lib.kda_forward_segmented_varlen_launches(T, H, dk, dv, chunk, DTYPES.get(dtype, dtype), num_seqs,
                                                      seg_len, PATHS[path])


def kda_forward_segmented(q, k, v, g, beta, S0=None, *, seg_len: int, chunk: int = 64, cu_seqlens=None, o=None,
                          S_T=None, return_state: bool = True, workspace=None, dev_status=None,
                          stream=None, path: str = "auto"):
    """kda_forward with every sequence cut into segments of ``seg_len`` tokens
    that run as independent units (segment pairs, a scan, a replay). Same shapes
    and results as kda_forward: B dense sequences, or (cu_seqlens, B = 1) a
    packed batch whose sequences longer than seg_len are cut."""
    _need(k, "k")
    dtype, dev = k.dtype, k.device
    if dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {dtype}")
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    _need(q, "q", dtype, (B, T, H, dk), dev)
    _need(g, "g", dtype, (B, T, H, dk), dev)
    _need(v, "v", dtype, (B, T, H, dv), dev)
    _need(beta, "beta", dtype, (B, T, H), dev)
    N = B
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        N = cu_seqlens.numel() - 1
    if S0 is not None:
        _need(S0, "S0", torch.float32, (N, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dtype, device=dev)
    _need(o, "o", dtype, (B, T, H, dv), dev)
    if return_state and S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (N, H, dv, dk), dev)
    if cu_seqlens is not None:
        ws_need = kda_forward_segmented_varlen_workspace_size(T, H, dk, dv, chunk, dtype, N, seg_len)
    else:
        ws_need = kda_forward_segmented_workspace_size(B, T, H, dk, dv, chunk, dtype, seg_len)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("cu_seqlens needs B == 1")
        rc = _lib.kda_forward_segmented_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                               _ptr(S_T), T, H, dk, dv, int(chunk), DTYPES[dtype],
                                               _ptr(cu_seqlens), N, int(seg_len), _ptr(workspace), ws_bytes,
                                               _ptr(dev_status), _stream_handle(stream, dev), PATHS[path])
    else:
        rc = _lib.kda_forward_segmented(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                        _ptr(S_T), B, T, H, dk, dv, int(chunk), DTYPES[dtype], int(seg_len),
                                        _ptr(workspace), ws_bytes, _ptr(dev_status),
                                        _stream_handle(stream, dev), PATHS[path])
    if rc != KDA_OK:
        raise KdaError(rc, "kda_forward_segmented")
    return o, S_T


def kda_decode_step(q, k, v, g, beta, S, o=None, *, stream=None, fuse: int = 0):
    """One decode token per request. q, k, g ``[N, H, dk]``; v ``[N, H, dv]``;
    beta ``[N, H]``; S ``[N, H, dv, dk]`` fp32 updated in place. ``fuse``:
    KDA_FUSE_* bits. Returns o."""
    _need(k, "k")
    dtype, dev = k.dtype, k.device
    N, H, dk = k.shape
    dv = v.shape[-1]
    _need(q, "q", dtype, (N, H, dk), dev)
    _need(g, "g", dtype, (N, H, dk), dev)
    _need(v, "v", dtype, (N, H, dv), dev)
    _need(beta, "beta", dtype, (N, H), dev)
    _need(S, "S", torch.float32, (N, H, dv, dk), dev)
    if o is None:
        o = torch.empty((N, H, dv), dtype=dtype, device=dev)
    _need(o, "o", dtype, (N, H, dv), dev)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o), N, H, dk, dv, DTYPES[dtype],
            _stream_handle(stream, dev))
    rc = _lib.kda_decode_step_fused(*args, int(fuse)) if fuse else _lib.kda_decode_step(*args)
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_step")
    return o


def kda_decode_multi(q, k, v, g, beta, S, o=None, *, n_accept=None, outputs: bool = True, dev_status=None,
                     stream=None):
    """T tokens per request from the states S (fp32 ``[N, H, dv, dk]``): outputs
    of all T tokens, and the state after the first ``n_accept[n]`` tokens written
    back in place (int32 ``[N]`` on the device; None = all T; 0 = untouched).
    q, k, g ``[N, T, H, dk]``; v ``[N, T, H, dv]``; beta ``[N, T, H]``.
    Returns o ``[N, T, H, dv]`` (None when ``outputs`` is False and o is None)."""
    _need(k, "k")
    dtype, dev = k.dtype, k.device
    N, T, H, dk = k.shape
    dv = v.shape[-1]
    _need(q, "q", dtype, (N, T, H, dk), dev)
    _need(g, "g", dtype, (N, T, H, dk), dev)
    _need(v, "v", dtype, (N, T, H, dv), dev)
    _need(beta, "beta", dtype, (N, T, H), dev)
    _need(S, "S", torch.float32, (N, H, dv, dk), dev)
    if n_accept is not None:
        _need(n_accept, "n_accept", torch.int32, (N,), dev)
    if o is None and outputs:
        o = torch.empty((N, T, H, dv), dtype=dtype, device=dev)
    if o is not None:
        _need(o, "o", dtype, (N, T, H, dv), dev)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, None, dev)
    rc = _lib.kda_decode_multi(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                               _ptr(n_accept), N, T, H, dk, dv, DTYPES[dtype], _ptr(dev_status),
                               _stream_handle(stream, dev))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_multi")
    return o


def kda_forward_snapshots(q, k, v, g, beta, S0=None, *, snap_every: int, chunk: int = 64, o=None,
                          S_T=None, S_snap=None, workspace=None, dev_status=None, stream=None,
                          path: str = "auto"):
    """kda_forward on B dense sequences that also returns the state every
    ``snap_every`` tokens: S_snap fp32 ``[B, T // snap_every, H, dv, dk]`` (slot p =
    the state after (p + 1) * snap_every tokens, usable as S0 of one sequence).
    Returns ``(o, S_T, S_snap)``."""
    _need(k, "k")
    dtype, dev = k.dtype, k.device
    if dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {dtype}")
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    _need(q, "q", dtype, (B, T, H, dk), dev)
    _need(g, "g", dtype, (B, T, H, dk), dev)
    _need(v, "v", dtype, (B, T, H, dv), dev)
    _need(beta, "beta", dtype, (B, T, H), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dtype, device=dev)
    _need(o, "o", dtype, (B, T, H, dv), dev)
    if S_T is None:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    _need(S_T, "S_T", torch.float32, (B, H, dv, dk), dev)
    nsnap = T // snap_every if snap_every > 0 else 0
    if S_snap is None:
        S_snap = torch.empty((B, nsnap, H, dv, dk), dtype=torch.float32, device=dev)
    _need(S_snap, "S_snap", torch.float32, (B, nsnap, H, dv, dk), dev)
    if workspace is None and path != "tc_single":  # the split form where it applies (the single form without)
        n = kda_forward_workspace_size(B, T, H, dk, dv, chunk, B, dtype, path=path)
        if n > 0:
            workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.kda_forward_snapshots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                    _ptr(S_T), _ptr(S_snap) if nsnap > 0 else None, int(snap_every), B, T, H,
                                    dk, dv, int(chunk), DTYPES[dtype], _ptr(workspace), ws_bytes,
                                    _ptr(dev_status), _stream_handle(stream, dev), PATHS[path])
    if rc != KDA_OK:
        raise KdaError(rc, "kda_forward_snapshots")
    return o, S_T, S_snap


def kda_segment_pair(q, k, v, g, beta, *, chunk: int = 64, dev_status=None, stream=None, path: str = "auto"):
    """KCP pair of each of B dense sequences: M fp32 ``[B, H, dk, dk]`` (the transition,
    stored like a state with dv = dk) and Z fp32 ``[B, H, dv, dk]`` (the local state)."""
    _need(k, "k")
    dtype, dev = k.dtype, k.device
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    _need(q, "q", dtype, (B, T, H, dk), dev)
    _need(g, "g", dtype, (B, T, H, dk), dev)
    _need(v, "v", dtype, (B, T, H, dv), dev)
    _need(beta, "beta", dtype, (B, T, H), dev)
    M = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    Z = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    rc = _lib.kda_segment_pair(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(M), _ptr(Z), B, T, H, dk,
                               dv, int(chunk), DTYPES[dtype], _ptr(dev_status), _stream_handle(stream, dev),
                               PATHS[path])
    if rc != KDA_OK:
        raise KdaError(rc, "kda_segment_pair")
    return M, Z


def kda_kcp_scan(S0, M, Z, *, stream=None):
    """Incoming state of every segment from the segments' pairs: M ``[B, P, H, dk, dk]``,
    Z ``[B, P, H, dv, dk]``, S0 ``[B, H, dv, dk]`` or None. Returns (S_in
    ``[B, P, H, dv, dk]``, S_T ``[B, H, dv, dk]``), fp32."""
    _need(M, "M", torch.float32)
    B, P, H, dk, _ = M.shape
    dv = Z.shape[3]
    dev = M.device
    _need(Z, "Z", torch.float32, (B, P, H, dv, dk), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    S_in = torch.empty((B, P, H, dv, dk), dtype=torch.float32, device=dev)
    S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    rc = _lib.kda_kcp_scan(_ptr(S0), _ptr(M), _ptr(Z), _ptr(S_in), _ptr(S_T), B, P, H, dk, dv,
                           _stream_handle(stream, dev))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_kcp_scan")
    return S_in, S_T


def kda_selftest_wait_timeout(dev_status, max_cycles: int = 20_000_000, *, stream=None):
    """Run the bounded-wait self-test (a wait that must run out); the caller reads
    dev_status (int32 on the device) after synchronising: KDA_ERR_TIMEOUT."""
    _need(dev_status, "dev_status", torch.int32)
    rc = _lib.kda_selftest_wait_timeout(_ptr(dev_status), int(max_cycles), _stream_handle(stream, dev_status.device))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_selftest_wait_timeout")
