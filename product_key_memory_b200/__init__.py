"""Python binding of libpkm.so, the B200 (sm_100a) product-key memory library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. The functions carry the names of the C entry points in include/pkm.h.
PyTorch supplies device memory and the current stream.

The library must have been built (``python product_key_memory_b200/build.py``);
importing this package raises if libpkm.so is missing. There is no CPU path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# PKM_LIBRARY selects another build of the library (the timeout test build).
LIB_PATH = os.environ.get("PKM_LIBRARY") or os.path.join(_HERE, "libpkm.so")

PKM_F32, PKM_BF16 = 0, 1
PKM_OK = 0
PKM_OPT_PATH, PKM_OPT_SUBBATCHES = 0, 1
PKM_PATH_AUTO, PKM_PATH_TC, PKM_PATH_SIMT, PKM_PATH_SMALL_FUSED, PKM_PATH_SMALL_SPLIT = range(5)
_PATHS = {"auto": PKM_PATH_AUTO, "tc": PKM_PATH_TC, "simt": PKM_PATH_SIMT,
          "small_fused": PKM_PATH_SMALL_FUSED, "small_split": PKM_PATH_SMALL_SPLIT}
_STATUS = {0: "PKM_OK", -1: "PKM_ERR_INVALID_ARG", -2: "PKM_ERR_UNSUPPORTED",
           -3: "PKM_ERR_WORKSPACE", -4: "PKM_ERR_CUDA", -5: "PKM_ERR_DEVICE"}

EXPORTED = ("pkm_workspace_size", "pkm_forward", "pkm_backward_values", "pkm_device_status",
            "pkm_trace_enable", "pkm_trace_read", "pkm_status_string",
            "pkm_backward_values_noalloc", "pkm_slot_usage", "pkm_backward",
            "pkm_forward_train", "pkm_backward_train", "pkm_set_option", "pkm_get_option")


class PKMError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__("%s returned %s (%d): %s" % (fn, _STATUS.get(code, "?"), code,
                                                      pkm_status_string(code)))
        self.code = code


class pkm_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("d_model", ctypes.c_int32), ("H", ctypes.c_int32),
                ("dq", ctypes.c_int32), ("n", ctypes.c_int32), ("k", ctypes.c_int32),
                ("v", ctypes.c_int32), ("dtype", ctypes.c_int32), ("bn_eps", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libpkm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("%s not built: run python product_key_memory_b200/build.py"
                              % os.path.basename(LIB_PATH))
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        S = ctypes.POINTER(pkm_shape)
        L.pkm_workspace_size.argtypes = [S, ctypes.c_int]
        L.pkm_workspace_size.restype = ctypes.c_size_t
        L.pkm_forward.argtypes = [S] + [P] * 13 + [ctypes.c_size_t, P]
        L.pkm_forward.restype = ctypes.c_int
        L.pkm_backward_values.argtypes = [S] + [P] * 7 + [ctypes.c_size_t, P]
        L.pkm_backward_values.restype = ctypes.c_int
        L.pkm_backward.argtypes = [S] + [P] * 19 + [ctypes.c_size_t, P]
        L.pkm_backward.restype = ctypes.c_int
        L.pkm_backward_train.argtypes = [S] + [P] * 19 + [ctypes.c_size_t, P]
        L.pkm_backward_train.restype = ctypes.c_int
        L.pkm_forward_train.argtypes = [S] + [P] * 6 + [ctypes.c_float] + [P] * 9 + [
            ctypes.c_size_t, P]
        L.pkm_forward_train.restype = ctypes.c_int
        L.pkm_backward_values_noalloc.argtypes = [S] + [P] * 6 + [P]
        L.pkm_backward_values_noalloc.restype = ctypes.c_int
        L.pkm_slot_usage.argtypes = [S, P, P, P, ctypes.c_size_t, P]
        L.pkm_slot_usage.restype = ctypes.c_int
        L.pkm_device_status.argtypes = [P, P]
        L.pkm_device_status.restype = ctypes.c_int
        L.pkm_trace_enable.argtypes = [ctypes.c_int]
        L.pkm_trace_enable.restype = ctypes.c_int
        L.pkm_trace_read.argtypes = [ctypes.c_int, P, ctypes.c_int, P, P]
        L.pkm_trace_read.restype = ctypes.c_int
        L.pkm_set_option.argtypes = [ctypes.c_int, ctypes.c_int]
        L.pkm_set_option.restype = ctypes.c_int
        L.pkm_get_option.argtypes = [ctypes.c_int]
        L.pkm_get_option.restype = ctypes.c_int
        L.pkm_status_string.argtypes = [ctypes.c_int]
        L.pkm_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


lib()  # fail loudly at import when the library is missing


def pkm_status_string(code: int) -> str:
    return lib().pkm_status_string(int(code)).decode()


def pkm_set_option(option: int, value: int) -> None:
    rc = lib().pkm_set_option(int(option), int(value))
    if rc != PKM_OK:
        raise PKMError("pkm_set_option", rc)


def pkm_get_option(option: int) -> int:
    rc = int(lib().pkm_get_option(int(option)))
    if rc < 0:
        raise PKMError("pkm_get_option", rc)
    return rc


class options:
    """Context manager that sets the library's implementation switches and restores
    them on exit: ``with options(path="simt"): ...`` (path: "auto", "tc", "simt",
    "small_fused" or "small_split"; subbatches: 1..4)."""

    def __init__(self, path: Optional[str] = None, subbatches: Optional[int] = None):
        self.want = {}
        if path is not None:
            self.want[PKM_OPT_PATH] = _PATHS[path]
        if subbatches is not None:
            self.want[PKM_OPT_SUBBATCHES] = int(subbatches)

    def __enter__(self):
        self.old = {o: pkm_get_option(o) for o in self.want}
        for o, v in self.want.items():
            pkm_set_option(o, v)
        return self

    def __exit__(self, *exc):
        for o, v in self.old.items():
            pkm_set_option(o, v)


def make_shape(B, d_model, H, dq, n, k, v, dtype, bn_eps=1e-5) -> pkm_shape:
    dt = dtype if isinstance(dtype, int) else (PKM_BF16 if dtype == torch.bfloat16 else PKM_F32)
    return pkm_shape(int(B), int(d_model), int(H), int(dq), int(n), int(k), int(v), dt,
                     float(bn_eps))


def pkm_workspace_size(shape: pkm_shape, for_backward: bool = False) -> int:
    return int(lib().pkm_workspace_size(ctypes.byref(shape), int(bool(for_backward))))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libpkm takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libpkm takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def alloc_workspace(shape: pkm_shape, for_backward: bool = False,
                    device=None) -> torch.Tensor:
    n = pkm_workspace_size(shape, for_backward)
    if n == 0:
        raise PKMError("pkm_workspace_size", -1)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def pkm_forward(x: torch.Tensor, W_q: torch.Tensor, bn_mean: torch.Tensor,
                bn_var: torch.Tensor, bn_gamma: torch.Tensor, bn_beta: torch.Tensor,
                subkeys: torch.Tensor, values: torch.Tensor, k: int, bn_eps: float = 1e-5,
                out: Optional[torch.Tensor] = None, indices: Optional[torch.Tensor] = None,
                weights: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                want_scores: bool = True, workspace: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor,
                                      Optional[torch.Tensor]]:
    """Run the PKM forward on the current CUDA stream.

    x [B][d_model], W_q [H*dq][d_model], BN vectors [H*dq] fp32, subkeys [H][2][n][dq/2],
    values [n*n][v] -- x, W_q, subkeys, values all fp32 or all bf16.
    Returns (out [B][v] fp32, indices [B][H][k] int32, weights [B][H][k] fp32,
    scores [B][H][k] fp32 or None). Missing outputs are allocated here.
    """
    B, d = x.shape
    H, two, n, half = subkeys.shape
    if two != 2:
        raise ValueError("subkeys must be [H][2][n][dq/2]")
    v = values.shape[1]
    shape = make_shape(B, d, H, 2 * half, n, k, v, x.dtype, bn_eps)
    dev = x.device
    if out is None:
        out = torch.empty(B, v, dtype=torch.float32, device=dev)
    if indices is None:
        indices = torch.empty(B, H, k, dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty(B, H, k, dtype=torch.float32, device=dev)
    if scores is None and want_scores:
        scores = torch.empty(B, H, k, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(shape, False, dev)
    rc = lib().pkm_forward(ctypes.byref(shape), _ptr(x), _ptr(W_q), _ptr(bn_mean), _ptr(bn_var),
                           _ptr(bn_gamma), _ptr(bn_beta), _ptr(subkeys), _ptr(values), _ptr(out),
                           _ptr(indices), _ptr(weights), _ptr(scores), _ptr(workspace),
                           workspace.numel(), _stream(stream))
    if rc != PKM_OK:
        raise PKMError("pkm_forward", rc)
    return out, indices, weights, scores


def pkm_backward_values(values: torch.Tensor, indices: torch.Tensor, weights: torch.Tensor,
                        grad_out: torch.Tensor, grad_values: torch.Tensor,
                        grad_scores: Optional[torch.Tensor], n: int,
                        workspace: Optional[torch.Tensor] = None, stream=None):
    """Sparse value backward. grad_values [n*n][v] fp32 is accumulated into;
    grad_scores [B][H][k] fp32 is overwritten (may be None)."""
    B, H, k = indices.shape
    v = values.shape[1]
    shape = make_shape(B, 0, H, 0, n, k, v, values.dtype)
    if workspace is None:
        workspace = alloc_workspace(shape, True, values.device)
    rc = lib().pkm_backward_values(ctypes.byref(shape), _ptr(values), _ptr(indices),
                                   _ptr(weights), _ptr(grad_out), _ptr(grad_values),
                                   _ptr(grad_scores), _ptr(workspace), workspace.numel(),
                                   _stream(stream))
    if rc != PKM_OK:
        raise PKMError("pkm_backward_values", rc)
    return grad_values, grad_scores


def pkm_forward_train(x: torch.Tensor, W_q: torch.Tensor, bn_running_mean: torch.Tensor,
                      bn_running_var: torch.Tensor, bn_gamma: torch.Tensor,
                      bn_beta: torch.Tensor, subkeys: torch.Tensor, values: torch.Tensor, k: int,
                      momentum: float = 0.1, bn_eps: float = 1e-5,
                      workspace: Optional[torch.Tensor] = None, stream=None):
    """Forward with BatchNorm in training mode. Updates bn_running_mean/var in place;
    returns (out, indices, weights, scores, batch_mean, batch_var)."""
    B, d = x.shape
    H, _, n, half = subkeys.shape
    v = values.shape[1]
    F = H * 2 * half
    shape = make_shape(B, d, H, 2 * half, n, k, v, x.dtype, bn_eps)
    dev = x.device
    if workspace is None:
        nb = int(lib().pkm_workspace_size(ctypes.byref(shape), 4))
        if nb == 0:
            raise PKMError("pkm_workspace_size", -1)
        workspace = torch.empty(nb, dtype=torch.uint8, device=dev)
    out = torch.empty(B, v, dtype=torch.float32, device=dev)
    idx = torch.empty(B, H, k, dtype=torch.int32, device=dev)
    wts = torch.empty(B, H, k, dtype=torch.float32, device=dev)
    scs = torch.empty(B, H, k, dtype=torch.float32, device=dev)
    bm = torch.empty(F, dtype=torch.float32, device=dev)
    bv = torch.empty(F, dtype=torch.float32, device=dev)
    rc = lib().pkm_forward_train(ctypes.byref(shape), _ptr(x), _ptr(W_q), _ptr(bn_running_mean),
                                 _ptr(bn_running_var), _ptr(bn_gamma), _ptr(bn_beta),
                                 ctypes.c_float(momentum), _ptr(subkeys), _ptr(values), _ptr(out),
                                 _ptr(idx), _ptr(wts), _ptr(scs), _ptr(bm), _ptr(bv),
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != PKM_OK:
        raise PKMError("pkm_forward_train", rc)
    return out, idx, wts, scs, bm, bv


def pkm_backward(x: torch.Tensor, W_q: torch.Tensor, bn_mean: torch.Tensor,
                 bn_var: torch.Tensor, bn_gamma: torch.Tensor, bn_beta: torch.Tensor,
                 subkeys: torch.Tensor, values: torch.Tensor, indices: torch.Tensor,
                 weights: torch.Tensor, grad_out: torch.Tensor, grads: dict,
                 bn_eps: float = 1e-5, workspace: Optional[torch.Tensor] = None, stream=None,
                 bn_training: bool = False):
    """Full backward of the layer with the forward's picks held fixed.

    ``grads`` maps any of x [B][d], W_q [H*dq][d], bn_gamma, bn_beta [H*dq],
    subkeys [H][2][n][dq/2], values [n*n][v], scores [B][H][k] to fp32 device
    tensors; missing entries are not computed. values is accumulated into, the
    others are overwritten. With bn_training, bn_mean / bn_var are the batch
    statistics pkm_forward_train returned (pkm_backward_train)."""
    B, d = x.shape
    H, _, n, half = subkeys.shape
    k = indices.shape[2]
    v = values.shape[1]
    shape = make_shape(B, d, H, 2 * half, n, k, v, x.dtype, bn_eps)
    if workspace is None:
        nb = int(lib().pkm_workspace_size(ctypes.byref(shape), 3))
        if nb == 0:
            raise PKMError("pkm_workspace_size", -1)
        workspace = torch.empty(nb, dtype=torch.uint8, device=x.device)
    g = grads
    fn = lib().pkm_backward_train if bn_training else lib().pkm_backward
    rc = fn(ctypes.byref(shape), _ptr(x), _ptr(W_q), _ptr(bn_mean), _ptr(bn_var),
            _ptr(bn_gamma), _ptr(bn_beta), _ptr(subkeys), _ptr(values), _ptr(indices),
            _ptr(weights), _ptr(grad_out), _ptr(g.get("x")), _ptr(g.get("W_q")),
            _ptr(g.get("bn_gamma")), _ptr(g.get("bn_beta")), _ptr(g.get("subkeys")),
            _ptr(g.get("values")), _ptr(g.get("scores")), _ptr(workspace), workspace.numel(),
            _stream(stream))
    if rc != PKM_OK:
        raise PKMError("pkm_backward_train" if bn_training else "pkm_backward", rc)
    return grads


def pkm_backward_values_noalloc(values: torch.Tensor, indices: torch.Tensor,
                                weights: torch.Tensor, grad_out: torch.Tensor,
                                grad_values: torch.Tensor, grad_scores: Optional[torch.Tensor],
                                n: int, stream=None):
    """pkm_backward_values with the library's fixed device scratch instead of a
    workspace (for callers that cannot allocate; limits in include/pkm.h)."""
    B, H, k = indices.shape
    v = values.shape[1]
    shape = make_shape(B, 0, H, 0, n, k, v, values.dtype)
    rc = lib().pkm_backward_values_noalloc(ctypes.byref(shape), _ptr(values), _ptr(indices),
                                           _ptr(weights), _ptr(grad_out), _ptr(grad_values),
                                           _ptr(grad_scores), _stream(stream))
    if rc != PKM_OK:
        raise PKMError("pkm_backward_values_noalloc", rc)
    return grad_values, grad_scores


def pkm_slot_usage(indices: torch.Tensor, n: int, hits: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Distinct slots among indices [B][H][k] (device int64 tensor of one element)."""
    B, H, k = indices.shape
    shape = make_shape(B, 0, H, 0, n, k, 8, PKM_F32)
    if hits is None:
        hits = torch.empty(1, dtype=torch.int64, device=indices.device)
    if workspace is None:
        nb = int(lib().pkm_workspace_size(ctypes.byref(shape), 2))
        if nb == 0:
            raise PKMError("pkm_workspace_size", -1)
        workspace = torch.empty(nb, dtype=torch.uint8, device=indices.device)
    rc = lib().pkm_slot_usage(ctypes.byref(shape), _ptr(indices), _ptr(hits), _ptr(workspace),
                              workspace.numel(), _stream(stream))
    if rc != PKM_OK:
        raise PKMError("pkm_slot_usage", rc)
    return hits


def pkm_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return (and clear) the workspace's device status."""
    return int(lib().pkm_device_status(_ptr(workspace), _stream(stream)))


def pkm_trace_enable(on: bool = True) -> None:
    """Record CUDA events at stage boundaries of every following call."""
    lib().pkm_trace_enable(int(bool(on)))


def pkm_trace_read(pass_: int = 0, max_stages: int = 4):
    """(per-stage milliseconds summed over traced calls, traced calls, kernel launches)
    for pass 0 (forward) or 1 (backward); waits for the events and resets."""
    ms = (ctypes.c_double * max_stages)()
    calls = ctypes.c_int64(0)
    launches = ctypes.c_int64(0)
    rc = lib().pkm_trace_read(int(pass_), ms, max_stages, ctypes.byref(calls),
                              ctypes.byref(launches))
    if rc != PKM_OK:
        raise PKMError("pkm_trace_read", rc)
    return list(ms), int(calls.value), int(launches.value)
