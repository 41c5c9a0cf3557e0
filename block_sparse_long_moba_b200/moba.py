"""Python binding of libmoba.so (ctypes): argument marshalling only.

Every step of the MoBA forward pass runs in the library's CUDA kernels; PyTorch only provides
device memory and the current stream. The functions mirror the C entry points of include/moba.h
and raise if the library is missing or a call fails — there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOBA_CHECKS=1 in the environment selects the build with device-side index checks
LIB_PATH = os.path.join(_HERE, "libmoba_checks.so" if os.environ.get("MOBA_CHECKS") == "1"
                        else "libmoba.so")

STATUS = {0: "MOBA_OK", -1: "MOBA_ERR_ARG", -2: "MOBA_ERR_UNSUPPORTED", -3: "MOBA_ERR_WORKSPACE",
          -4: "MOBA_ERR_CUDA", -5: "MOBA_ERR_DEVICE_CHECK", -6: "MOBA_ERR_TIMEOUT"}
KERNEL_CLASSES = ["centroid", "gate", "route_count", "route_scan", "route_scatter", "attention",
                  "merge", "plan", "densify", "decode", "bwd_dkdv", "bwd_dq", "bwd_aux"]

# every symbol include/moba.h declares
EXPORTS = ["moba_status_string", "moba_version", "moba_workspace_bytes", "moba_centroids",
           "moba_gate_topk", "moba_attn_fwd", "moba_device_status", "moba_timing_enable",
           "moba_timing_reset", "moba_timing_read", "moba_launch_count",
           "moba_attn_fwd_noalloc", "moba_noalloc_status", "moba_set_wait_limit_ns",
           "moba_centroids_kconv", "moba_attn_fwd_kconv", "moba_decode_workspace_bytes",
           "moba_decode_fwd", "moba_bwd_workspace_bytes", "moba_attn_bwd",
           "moba_set_diag_stall"]

NOALLOC_SCRATCH_BYTES = 64 << 20


class MobaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {STATUS.get(status, status)}")


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoba.so, or libmoba_checks.so when MOBA_CHECKS=1 (build them with
    `python -m block_sparse_long_moba_b200.build [--checks]`)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmoba.so not found at {path}; build it with "
                          "`python -m block_sparse_long_moba_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, L, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
    lib.moba_status_string.argtypes = [I]
    lib.moba_status_string.restype = ctypes.c_char_p
    lib.moba_version.restype = I
    lib.moba_workspace_bytes.argtypes = [I, P, I, I, I, I, I]
    lib.moba_workspace_bytes.restype = S
    lib.moba_centroids.argtypes = [P, P, P, I, I, I, I, P, P]
    lib.moba_centroids.restype = I
    lib.moba_gate_topk.argtypes = [P, P, P, P, I, I, I, I, I, I, P, P]
    lib.moba_gate_topk.restype = I
    lib.moba_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, P, P, S, P]
    lib.moba_attn_fwd.restype = I
    lib.moba_device_status.argtypes = [P, P]
    lib.moba_device_status.restype = I
    lib.moba_timing_enable.argtypes = [I]
    lib.moba_timing_enable.restype = I
    lib.moba_timing_reset.restype = I
    lib.moba_timing_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(L), I]
    lib.moba_timing_read.restype = I
    lib.moba_launch_count.restype = L
    lib.moba_attn_fwd_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P, P, P]
    lib.moba_attn_fwd_noalloc.restype = I
    lib.moba_centroids_kconv.argtypes = [P, P, I, P, P, I, I, I, I, P, P]
    lib.moba_centroids_kconv.restype = I
    lib.moba_attn_fwd_kconv.argtypes = [P, P, P, P, I, P, P, I, I, I, I, I, I, F, P, P, P, P, S, P]
    lib.moba_attn_fwd_kconv.restype = I
    lib.moba_decode_workspace_bytes.argtypes = [I, P, P, I, I, I, I, I]
    lib.moba_decode_workspace_bytes.restype = S
    lib.moba_decode_fwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, P, P, S,
                                    P]
    lib.moba_decode_fwd.restype = I
    lib.moba_bwd_workspace_bytes.argtypes = [I, P, I, I, I, I, I]
    lib.moba_bwd_workspace_bytes.restype = S
    lib.moba_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, P, S, P]
    lib.moba_attn_bwd.restype = I
    lib.moba_noalloc_status.argtypes = [P]
    lib.moba_noalloc_status.restype = I
    lib.moba_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.moba_set_wait_limit_ns.restype = ctypes.c_ulonglong
    lib.moba_set_diag_stall.argtypes = [I]
    lib.moba_set_diag_stall.restype = I
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        raise MobaError(status, what)


_ANY_DEVICE = object()  # the device is checked separately (_current_device)


def _bad(what: str, why: str):
    raise MobaError(-1, f"{what}: {why}")


def _want(what: str, name: str, t: Optional[torch.Tensor], dtype, shape=None, device=None):
    """Checks one tensor argument before its pointer reaches the library: the kernels trust the
    layout (dtype, contiguity, shape) and launch on the current device, so a mismatch here would
    otherwise read or write the wrong memory."""
    if t is None:
        _bad(what, f"{name} is required")
    if not torch.is_tensor(t):
        _bad(what, f"{name} must be a torch tensor")
    if t.dtype != dtype:
        _bad(what, f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        _bad(what, f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        _bad(what, f"{name} must be contiguous")
    if device is None:
        if t.device.type != "cuda":
            _bad(what, f"{name} must be a CUDA tensor, got {t.device}")
    elif device is not _ANY_DEVICE and t.device != device:
        _bad(what, f"{name} is on {t.device}, the call runs on {device}")


def _current_device(what: str, t: torch.Tensor) -> torch.device:
    if t.device.type != "cuda":
        _bad(what, f"tensors must be CUDA tensors, got {t.device}")
    cur = torch.device("cuda", torch.cuda.current_device())
    if t.device != cur:
        _bad(what, f"tensors are on {t.device} but the current device is {cur}")
    return cur


def _want_cu(what: str, cu_seqlens: torch.Tensor, nseq: int, device):
    _want(what, "cu_seqlens", cu_seqlens, torch.int32, (nseq + 1,), device)


def _host_cu(cu_seqlens_host) -> Tuple[ctypes.Array, int]:
    vals = [int(x) for x in (cu_seqlens_host.tolist() if torch.is_tensor(cu_seqlens_host)
                             else cu_seqlens_host)]
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return arr, len(vals) - 1


def num_blocks(cu_seqlens_host: Sequence[int], block_size: int) -> int:
    cu = [int(x) for x in cu_seqlens_host]
    return sum((cu[s + 1] - cu[s] + block_size - 1) // block_size for s in range(len(cu) - 1))


def moba_workspace_bytes(cu_seqlens_host, hq: int, hkv: int, d: int, block_size: int,
                         topk: int) -> int:
    arr, nseq = _host_cu(cu_seqlens_host)
    return int(load_library().moba_workspace_bytes(nseq, arr, hq, hkv, d, block_size, topk))


def moba_centroids(k: torch.Tensor, cu_seqlens: torch.Tensor, cu_seqlens_host, block_size: int,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Block centroids [NB, Hkv, d] fp32 of bf16 keys [T, Hkv, d]."""
    what = "moba_centroids"
    arr, nseq = _host_cu(cu_seqlens_host)
    if not torch.is_tensor(k) or k.dim() != 3:
        _bad(what, "k must be a [T, Hkv, d] tensor")
    T, hkv, d = k.shape
    _want(what, "k", k, torch.bfloat16, None, _ANY_DEVICE)
    dev = _current_device(what, k)
    _want_cu(what, cu_seqlens, nseq, dev)
    nb = num_blocks(list(arr), block_size)
    if out is None:
        out = torch.empty((nb, hkv, d), dtype=torch.float32, device=k.device)
    _want(what, "out", out, torch.float32, (nb, hkv, d), dev)
    st = load_library().moba_centroids(_ptr(k), _ptr(cu_seqlens), arr, nseq, hkv, d, block_size,
                                       _ptr(out), _stream(stream))
    _check(st, "moba_centroids")
    return out


def moba_centroids_kconv(k: torch.Tensor, conv_w: torch.Tensor, cu_seqlens: torch.Tensor,
                         cu_seqlens_host, block_size: int, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """Centroids [NB, Hkv, d] fp32 of keys passed through the in-block short convolution with
    weights conv_w [W, Hkv, d] fp32."""
    what = "moba_centroids_kconv"
    arr, nseq = _host_cu(cu_seqlens_host)
    if not torch.is_tensor(k) or k.dim() != 3 or not torch.is_tensor(conv_w) or conv_w.dim() != 3:
        _bad(what, "k must be [T, Hkv, d] and conv_w [W, Hkv, d]")
    T, hkv, d = k.shape
    _want(what, "k", k, torch.bfloat16, None, _ANY_DEVICE)
    dev = _current_device(what, k)
    _want(what, "conv_w", conv_w, torch.float32, (conv_w.shape[0], hkv, d), dev)
    _want_cu(what, cu_seqlens, nseq, dev)
    nb = num_blocks(list(arr), block_size)
    if out is None:
        out = torch.empty((nb, hkv, d), dtype=torch.float32, device=k.device)
    _want(what, "out", out, torch.float32, (nb, hkv, d), dev)
    st = load_library().moba_centroids_kconv(_ptr(k), _ptr(conv_w), conv_w.shape[0],
                                             _ptr(cu_seqlens), arr, nseq, hkv, d, block_size,
                                             _ptr(out), _stream(stream))
    _check(st, what)
    return out


def moba_gate_topk(q: torch.Tensor, centroids: torch.Tensor, cu_seqlens: torch.Tensor,
                   cu_seqlens_host, block_size: int, topk: int,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Routing [Hq, T, topk] int32 (ascending local block ids, -1 padded)."""
    what = "moba_gate_topk"
    arr, nseq = _host_cu(cu_seqlens_host)
    if not torch.is_tensor(q) or q.dim() != 3 or not torch.is_tensor(centroids) or \
            centroids.dim() != 3:
        _bad(what, "q must be [T, Hq, d] and centroids [NB, Hkv, d]")
    T, hq, d = q.shape
    hkv = centroids.shape[1]
    _want(what, "q", q, torch.bfloat16, None, _ANY_DEVICE)
    dev = _current_device(what, q)
    _want(what, "centroids", centroids, torch.float32,
          (num_blocks(list(arr), block_size), hkv, d), dev)
    _want_cu(what, cu_seqlens, nseq, dev)
    if out is None:
        out = torch.empty((hq, T, topk), dtype=torch.int32, device=q.device)
    _want(what, "out", out, torch.int32, (hq, T, topk), dev)
    st = load_library().moba_gate_topk(_ptr(q), _ptr(centroids), _ptr(cu_seqlens), arr, nseq, hq,
                                       hkv, d, block_size, topk, _ptr(out), _stream(stream))
    _check(st, "moba_gate_topk")
    return out


def _check_qkv(what, q, k, v, cu_seqlens, nseq):
    """q [T, Hq, d], k and v [T, Hkv, d], all bf16, contiguous, on the current device."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not torch.is_tensor(t) or t.dim() != 3:
            _bad(what, f"{name} must be a 3-D tensor")
    T, hq, d = q.shape
    hkv = k.shape[1]
    _want(what, "q", q, torch.bfloat16, None, _ANY_DEVICE)
    dev = _current_device(what, q)
    _want(what, "k", k, torch.bfloat16, (T, hkv, d), dev)
    _want(what, "v", v, torch.bfloat16, (T, hkv, d), dev)
    _want_cu(what, cu_seqlens, nseq, dev)
    return dev, T, hq, hkv, d


def moba_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                  cu_seqlens_host, block_size: int, topk: int, scale: Optional[float] = None,
                  block_idx_in: Optional[torch.Tensor] = None,
                  block_idx_out: Optional[torch.Tensor] = None,
                  o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None):
    """MoBA forward: returns (o [T,Hq,d] bf16, lse [Hq,T] fp32). Buffers may be passed in."""
    what = "moba_attn_fwd"
    arr, nseq = _host_cu(cu_seqlens_host)
    dev, T, hq, hkv, d = _check_qkv(what, q, k, v, cu_seqlens, nseq)
    if scale is None:
        scale = d ** -0.5
    for name, t in (("block_idx_in", block_idx_in), ("block_idx_out", block_idx_out)):
        if t is not None:
            _want(what, name, t, torch.int32, (hq, T, topk), dev)
    lib = load_library()
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=q.device)
    _want(what, "o", o, torch.bfloat16, (T, hq, d), dev)
    _want(what, "lse", lse, torch.float32, (hq, T), dev)
    if workspace is not None:
        _want(what, "workspace", workspace, torch.uint8, None, dev)
    if workspace is None:
        nbytes = int(lib.moba_workspace_bytes(nseq, arr, hq, hkv, d, block_size, topk))
        if nbytes == 0 and T > 0:
            raise MobaError(-1, "moba_workspace_bytes")
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    st = lib.moba_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), arr, nseq, hq, hkv, d,
                           block_size, topk, ctypes.c_float(scale), _ptr(block_idx_in),
                           _ptr(block_idx_out), _ptr(o), _ptr(lse), _ptr(workspace),
                           ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(st, "moba_attn_fwd")
    return o, lse


def moba_attn_fwd_kconv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                        conv_w: torch.Tensor, cu_seqlens: torch.Tensor, cu_seqlens_host,
                        block_size: int, topk: int, scale: Optional[float] = None,
                        block_idx_out: Optional[torch.Tensor] = None,
                        o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None):
    """MoBA forward with the routing computed on short-convolved keys (conv_w [W, Hkv, d] fp32);
    returns (o, lse)."""
    what = "moba_attn_fwd_kconv"
    arr, nseq = _host_cu(cu_seqlens_host)
    dev, T, hq, hkv, d = _check_qkv(what, q, k, v, cu_seqlens, nseq)
    if not torch.is_tensor(conv_w) or conv_w.dim() != 3:
        _bad(what, "conv_w must be [W, Hkv, d]")
    _want(what, "conv_w", conv_w, torch.float32, (conv_w.shape[0], hkv, d), dev)
    if scale is None:
        scale = d ** -0.5
    if block_idx_out is not None:
        _want(what, "block_idx_out", block_idx_out, torch.int32, (hq, T, topk), dev)
    lib = load_library()
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=q.device)
    _want(what, "o", o, torch.bfloat16, (T, hq, d), dev)
    _want(what, "lse", lse, torch.float32, (hq, T), dev)
    if workspace is None:
        nbytes = int(lib.moba_workspace_bytes(nseq, arr, hq, hkv, d, block_size, topk))
        if nbytes == 0 and T > 0:
            raise MobaError(-1, "moba_workspace_bytes")
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    _want(what, "workspace", workspace, torch.uint8, None, dev)
    st = lib.moba_attn_fwd_kconv(_ptr(q), _ptr(k), _ptr(v), _ptr(conv_w), conv_w.shape[0],
                                 _ptr(cu_seqlens), arr, nseq, hq, hkv, d, block_size, topk,
                                 ctypes.c_float(scale), _ptr(block_idx_out), _ptr(o), _ptr(lse),
                                 _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                 _stream(stream))
    _check(st, what)
    return o, lse


def moba_decode_workspace_bytes(cu_seqlens_host, cu_seqlens_q_host, hq: int, hkv: int, d: int,
                                block_size: int, topk: int) -> int:
    arr, nseq = _host_cu(cu_seqlens_host)
    arq, nq = _host_cu(cu_seqlens_q_host)
    if nq != nseq:
        _bad("moba_decode_workspace_bytes", "cu_seqlens_q must have nseq + 1 entries")
    return int(load_library().moba_decode_workspace_bytes(nseq, arr, arq, hq, hkv, d, block_size,
                                                          topk))


def moba_decode_fwd(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                    centroids: Optional[torch.Tensor], cu_seqlens: torch.Tensor, cu_seqlens_host,
                    cu_seqlens_q: torch.Tensor, cu_seqlens_q_host, block_size: int, topk: int,
                    scale: Optional[float] = None, block_idx_in: Optional[torch.Tensor] = None,
                    block_idx_out: Optional[torch.Tensor] = None,
                    o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None):
    """MoBA over the newest rows of a KV cache (decode: one row per sequence). q [Tq, Hq, d] are
    the last n_s tokens of each sequence (cu_seqlens_q); returns (o [Tq, Hq, d], lse [Hq, Tq])."""
    what = "moba_decode_fwd"
    arr, nseq = _host_cu(cu_seqlens_host)
    arq, nq = _host_cu(cu_seqlens_q_host)
    if nq != nseq:
        _bad(what, "cu_seqlens_q must have nseq + 1 entries")
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        if not torch.is_tensor(t) or t.dim() != 3:
            _bad(what, f"{name} must be a 3-D tensor")
    Tq, hq, d = q.shape
    T, hkv = k_cache.shape[0], k_cache.shape[1]
    _want(what, "q", q, torch.bfloat16, None, _ANY_DEVICE)
    dev = _current_device(what, q)
    _want(what, "k_cache", k_cache, torch.bfloat16, (T, hkv, d), dev)
    _want(what, "v_cache", v_cache, torch.bfloat16, (T, hkv, d), dev)
    _want_cu(what, cu_seqlens, nseq, dev)
    _want(what, "cu_seqlens_q", cu_seqlens_q, torch.int32, (nseq + 1,), dev)
    if centroids is not None:
        _want(what, "centroids", centroids, torch.float32,
              (num_blocks(list(arr), block_size), hkv, d), dev)
    elif block_idx_in is None:
        _bad(what, "centroids are required unless a routing is given")
    for name, t in (("block_idx_in", block_idx_in), ("block_idx_out", block_idx_out)):
        if t is not None:
            _want(what, name, t, torch.int32, (hq, Tq, topk), dev)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((hq, Tq), dtype=torch.float32, device=q.device)
    _want(what, "o", o, torch.bfloat16, (Tq, hq, d), dev)
    _want(what, "lse", lse, torch.float32, (hq, Tq), dev)
    if workspace is None:
        nbytes = int(lib.moba_decode_workspace_bytes(nseq, arr, arq, hq, hkv, d, block_size, topk))
        if nbytes == 0 and Tq > 0:
            raise MobaError(-1, "moba_decode_workspace_bytes")
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    _want(what, "workspace", workspace, torch.uint8, None, dev)
    st = lib.moba_decode_fwd(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(centroids),
                             _ptr(cu_seqlens), arr, _ptr(cu_seqlens_q), arq, nseq, hq, hkv, d,
                             block_size, topk, ctypes.c_float(scale), _ptr(block_idx_in),
                             _ptr(block_idx_out), _ptr(o), _ptr(lse), _ptr(workspace),
                             ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(st, what)
    return o, lse


def moba_bwd_workspace_bytes(cu_seqlens_host, hq: int, hkv: int, d: int, block_size: int,
                             topk: int) -> int:
    arr, nseq = _host_cu(cu_seqlens_host)
    return int(load_library().moba_bwd_workspace_bytes(nseq, arr, hq, hkv, d, block_size, topk))


def moba_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                  lse: torch.Tensor, d_o: torch.Tensor, block_idx: torch.Tensor,
                  cu_seqlens: torch.Tensor, cu_seqlens_host, block_size: int, topk: int,
                  scale: Optional[float] = None, dq: Optional[torch.Tensor] = None,
                  dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None):
    """Gradients (dq, dk, dv) of the routed attention with the routing held fixed; o and lse are
    the forward pass's outputs and block_idx the routing it used."""
    what = "moba_attn_bwd"
    arr, nseq = _host_cu(cu_seqlens_host)
    dev, T, hq, hkv, d = _check_qkv(what, q, k, v, cu_seqlens, nseq)
    _want(what, "o", o, torch.bfloat16, (T, hq, d), dev)
    _want(what, "d_o", d_o, torch.bfloat16, (T, hq, d), dev)
    _want(what, "lse", lse, torch.float32, (hq, T), dev)
    _want(what, "block_idx", block_idx, torch.int32, (hq, T, topk), dev)
    if scale is None:
        scale = d ** -0.5
    lib = load_library()
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _want(what, "dq", dq, torch.bfloat16, (T, hq, d), dev)
    _want(what, "dk", dk, torch.bfloat16, (T, hkv, d), dev)
    _want(what, "dv", dv, torch.bfloat16, (T, hkv, d), dev)
    if workspace is None:
        nbytes = int(lib.moba_bwd_workspace_bytes(nseq, arr, hq, hkv, d, block_size, topk))
        if nbytes == 0 and T > 0:
            raise MobaError(-1, "moba_bwd_workspace_bytes")
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    _want(what, "workspace", workspace, torch.uint8, None, dev)
    st = lib.moba_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o),
                           _ptr(block_idx), _ptr(cu_seqlens), arr, nseq, hq, hkv, d, block_size,
                           topk, ctypes.c_float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                           _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(st, what)
    return dq, dk, dv


def moba_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          cu_seqlens: torch.Tensor, cu_seqlens_host, block_size: int, topk: int,
                          scale: Optional[float] = None, o: Optional[torch.Tensor] = None,
                          lse: Optional[torch.Tensor] = None, stream=None):
    """moba_attn_fwd without a workspace: the library's static scratch array is used instead
    (for callers that cannot allocate device memory; see include/moba.h). The outputs may be
    passed in so that the call itself allocates nothing."""
    what = "moba_attn_fwd_noalloc"
    arr, nseq = _host_cu(cu_seqlens_host)
    dev, T, hq, hkv, d = _check_qkv(what, q, k, v, cu_seqlens, nseq)
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=q.device)
    _want(what, "o", o, torch.bfloat16, (T, hq, d), dev)
    _want(what, "lse", lse, torch.float32, (hq, T), dev)
    st = load_library().moba_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), arr,
                                              nseq, hq, hkv, d, block_size, topk,
                                              ctypes.c_float(scale), _ptr(o), _ptr(lse),
                                              _stream(stream))
    _check(st, "moba_attn_fwd_noalloc")
    return o, lse


def moba_device_status(workspace: torch.Tensor, stream=None) -> int:
    return int(load_library().moba_device_status(_ptr(workspace), _stream(stream)))


def moba_noalloc_status(stream=None) -> int:
    """Status word of the last moba_attn_fwd_noalloc call on the current device (synchronises)."""
    return int(load_library().moba_noalloc_status(_stream(stream)))


def set_wait_limit_ns(ns: int) -> int:
    """Diagnostics: limit of one pipeline wait in the attention kernel (0 = built-in 2 s);
    returns the previous limit."""
    return int(load_library().moba_set_wait_limit_ns(ctypes.c_ulonglong(int(ns))))


def set_diag_stall(on: bool) -> bool:
    """Diagnostics: make the attention kernel's MMA issuer wait on a barrier nothing arrives on
    (so that a short wait limit runs out); returns the previous setting."""
    return bool(load_library().moba_set_diag_stall(1 if on else 0))


def timing_enable(on: bool = True):
    load_library().moba_timing_enable(1 if on else 0)


def timing_reset():
    load_library().moba_timing_reset()


def timing_read() -> dict:
    lib = load_library()
    n = len(KERNEL_CLASSES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    r = lib.moba_timing_read(ms, cnt, n)
    if r < 0:
        raise MobaError(r, "moba_timing_read")
    return {KERNEL_CLASSES[i]: (float(ms[i]), int(cnt[i])) for i in range(n)}


def launch_count() -> int:
    return int(load_library().moba_launch_count())
