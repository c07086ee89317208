"""fp64 CPU oracle for the product-key memory layer (ctypes binding of pkm_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The CUDA library never imports
this package, and this package imports nothing from the CUDA library.

Every function takes and returns CPU tensors/arrays. bf16 tensors are handed to
the C code as their raw bit patterns, which it widens exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpkm_oracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile pkm_oracle.c with gcc (plain -O2, IEEE arithmetic, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.pkm_oracle_forward.argtypes = [_I64, _I, _I, _I, _I, _I, _I, _I, _D] + [_P] * 14 + [_I]
        L.pkm_oracle_forward.restype = _I
        L.pkm_oracle_flat_topk.argtypes = [_I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I]
        L.pkm_oracle_flat_topk.restype = _I
        L.pkm_oracle_finish.argtypes = [_I64, _I, _I, _I, _I, _P, _P, _P, _P, _P]
        L.pkm_oracle_finish.restype = _I
        L.pkm_oracle_backward.argtypes = [_I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]
        L.pkm_oracle_backward.restype = _I
        L.pkm_oracle_forward_train.argtypes = ([_I64, _I, _I, _I, _I, _I, _I, _I, _D, _D]
                                               + [_P] * 18 + [_I])
        L.pkm_oracle_forward_train.restype = _I
        L.pkm_oracle_backward_full.argtypes = [_I64, _I, _I, _I, _I, _I, _I, _I, _D, _I] + [_P] * 17
        L.pkm_oracle_backward_full.restype = _I
        L.pkm_oracle_slot_usage.argtypes = [_I64, _P, _I64, _P]
        L.pkm_oracle_slot_usage.restype = _I64
        _lib = L
    return _lib


def _raw(t: torch.Tensor):
    """(numpy array holding the bytes, dtype code) for an fp32 or bf16 tensor."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), 1
    if t.dtype == torch.float32:
        return t.numpy(), 0
    raise TypeError("oracle takes fp32 or bf16 tensors, got %s" % t.dtype)


def _f32(t: torch.Tensor) -> np.ndarray:
    return np.ascontiguousarray(t.detach().cpu().float().numpy())


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_P)


def forward(layer: dict, H: int, dq: int, n: int, k: int, eps: float = 1e-5,
            want_q: bool = False, want_half: bool = False, want_out: bool = True,
            threads: int = 0) -> dict:
    """Product-key forward for every row of ``layer['x']``.

    Returns numpy arrays: out [B][v] f64, indices [B][H][k] i32 (flat slot i*n+j),
    weights [B][H][k] f64, scores [B][H][k] f64, and optionally q [B][H*dq] and
    half [B][H][2][n] (every per-half sub-key score).
    """
    x, dt = _raw(layer["x"])
    W, dt2 = _raw(layer["W_q"])
    C, dt3 = _raw(layer["subkeys"])
    V, dt4 = _raw(layer["values"])
    if len({dt, dt2, dt3, dt4}) != 1:
        raise TypeError("x, W_q, subkeys and values must share one dtype")
    B, d = x.shape
    v = V.shape[1]
    mean, var = _f32(layer["bn_mean"]), _f32(layer["bn_var"])
    gamma, beta = _f32(layer["bn_gamma"]), _f32(layer["bn_beta"])
    out = np.zeros((B, v)) if want_out else None
    idx = np.zeros((B, H, k), np.int32)
    w = np.zeros((B, H, k))
    s = np.zeros((B, H, k))
    q = np.zeros((B, H * dq)) if want_q else None
    half = np.zeros((B, H, 2, n)) if want_half else None
    rc = lib().pkm_oracle_forward(B, d, H, dq, n, k, v, dt, eps, _ptr(x), _ptr(W),
                                  _ptr(mean), _ptr(var), _ptr(gamma), _ptr(beta), _ptr(C),
                                  _ptr(V), _ptr(out), _ptr(idx), _ptr(w), _ptr(s), _ptr(q),
                                  _ptr(half), threads)
    if rc != 0:
        raise ValueError("pkm_oracle_forward rejected the sizes")
    return dict(out=out, indices=idx, weights=w, scores=s, q=q, half=half)


def forward_train(layer: dict, H: int, dq: int, n: int, k: int, eps: float = 1e-5,
                  momentum: float = 0.1, want_q: bool = False, want_half: bool = False,
                  threads: int = 0) -> dict:
    """Forward with BatchNorm in training mode: the batch's own statistics normalise
    it and the running statistics (layer['bn_mean'], layer['bn_var']) move towards
    them. Returns forward()'s arrays plus batch_mean, batch_var (biased) and
    running_mean, running_var (the updated running statistics), all fp64."""
    x, dt = _raw(layer["x"])
    W, _ = _raw(layer["W_q"])
    C, _ = _raw(layer["subkeys"])
    V, _ = _raw(layer["values"])
    B, d = x.shape
    v = V.shape[1]
    F = H * dq
    rm, rv = _f32(layer["bn_mean"]), _f32(layer["bn_var"])
    gamma, beta = _f32(layer["bn_gamma"]), _f32(layer["bn_beta"])
    r = dict(out=np.zeros((B, v)), indices=np.zeros((B, H, k), np.int32),
             weights=np.zeros((B, H, k)), scores=np.zeros((B, H, k)),
             q=np.zeros((B, F)) if want_q else None,
             half=np.zeros((B, H, 2, n)) if want_half else None,
             batch_mean=np.zeros(F), batch_var=np.zeros(F), running_mean=np.zeros(F),
             running_var=np.zeros(F))
    rc = lib().pkm_oracle_forward_train(
        B, d, H, dq, n, k, v, dt, eps, momentum, _ptr(x), _ptr(W), _ptr(rm), _ptr(rv),
        _ptr(gamma), _ptr(beta), _ptr(C), _ptr(V), _ptr(r["out"]), _ptr(r["indices"]),
        _ptr(r["weights"]), _ptr(r["scores"]), _ptr(r["q"]), _ptr(r["half"]),
        _ptr(r["batch_mean"]), _ptr(r["batch_var"]), _ptr(r["running_mean"]),
        _ptr(r["running_var"]), threads)
    if rc != 0:
        raise ValueError("pkm_oracle_forward_train rejected the sizes")
    return r


def flat_topk(q: np.ndarray, subkeys: torch.Tensor, H: int, dq: int, n: int, k: int,
              threads: int = 0):
    """Brute-force top-k over all n*n explicit keys (no per-half scores involved)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    C, dt = _raw(subkeys)
    B = q.shape[0]
    idx = np.zeros((B, H, k), np.int32)
    sc = np.zeros((B, H, k))
    rc = lib().pkm_oracle_flat_topk(B, H, dq, n, k, dt, _ptr(q), _ptr(C), _ptr(idx), _ptr(sc),
                                    threads)
    if rc != 0:
        raise ValueError("pkm_oracle_flat_topk rejected the sizes")
    return idx, sc


def finish(scores: np.ndarray, indices: np.ndarray, values: torch.Tensor):
    """Softmax of given kept scores and the weighted value sum over heads."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    V, dt = _raw(values)
    B, H, k = scores.shape
    v = V.shape[1]
    w = np.zeros((B, H, k))
    out = np.zeros((B, v))
    rc = lib().pkm_oracle_finish(B, H, k, v, dt, _ptr(scores), _ptr(indices), _ptr(V),
                                 _ptr(w), _ptr(out))
    if rc != 0:
        raise ValueError("pkm_oracle_finish rejected the sizes")
    return w, out


def backward(values: torch.Tensor, grad_out: torch.Tensor, indices: np.ndarray,
             weights: np.ndarray, row_slot: Optional[np.ndarray] = None,
             rows: Optional[int] = None):
    """Sparse value backward. Returns (grad_values [rows][v] f64, grad_scores [B][H][k]).

    ``row_slot`` maps each flat slot to a row of the returned table (-1 = skip);
    without it the table is dense over all slots.
    """
    V, dt = _raw(values)
    G, dt2 = _raw(grad_out)
    if dt != dt2:
        raise TypeError("values and grad_out must share one dtype")
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    weights = np.ascontiguousarray(weights, dtype=np.float64)
    B, H, k = indices.shape
    v = V.shape[1]
    if row_slot is None:
        rows = V.shape[0]
    else:
        row_slot = np.ascontiguousarray(row_slot, dtype=np.int64)
    gv = np.zeros((rows, v))
    gs = np.zeros((B, H, k))
    rc = lib().pkm_oracle_backward(B, H, k, v, dt, _ptr(V), _ptr(G), _ptr(indices),
                                   _ptr(weights), _ptr(row_slot), _ptr(gv), _ptr(gs))
    if rc != 0:
        raise ValueError("pkm_oracle_backward rejected the sizes")
    return gv, gs


def slot_usage(indices: np.ndarray, slots: int):
    """(distinct slots among the picks, number of picks outside [0, slots))."""
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    bad = ctypes.c_int64(0)
    n = lib().pkm_oracle_slot_usage(indices.size, _ptr(indices), int(slots), ctypes.byref(bad))
    if n < 0:
        raise ValueError("pkm_oracle_slot_usage rejected the sizes")
    return int(n), int(bad.value)


def backward_full(layer: dict, indices: np.ndarray, weights: np.ndarray,
                  grad_out: torch.Tensor, H: int, dq: int, n: int, k: int, eps: float = 1e-5,
                  bn_training: bool = False):
    """Gradients of L = <grad_out, out> with the picks held fixed. Returns a dict of
    fp64 arrays: x [B][d], W_q [H*dq][d], gamma, beta [H*dq], subkeys [H][2][n][dq/2],
    q [B][H*dq] (dL/dq). With bn_training the batch's own statistics (recomputed from
    the batch) normalised the forward and the gradient flows through them too;
    layer['bn_mean'] / ['bn_var'] are then not read."""
    x, dt = _raw(layer["x"])
    W, _ = _raw(layer["W_q"])
    C, _ = _raw(layer["subkeys"])
    V, _ = _raw(layer["values"])
    G, dtg = _raw(grad_out)
    if dtg != dt:
        raise TypeError("grad_out must have the layer's dtype")
    B, d = x.shape
    v = V.shape[1]
    F = H * dq
    mean, var = _f32(layer["bn_mean"]), _f32(layer["bn_var"])
    gamma, beta = _f32(layer["bn_gamma"]), _f32(layer["bn_beta"])
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    weights = np.ascontiguousarray(weights, dtype=np.float64)
    out = dict(x=np.zeros((B, d)), W_q=np.zeros((F, d)), gamma=np.zeros(F), beta=np.zeros(F),
               subkeys=np.zeros((H, 2, n, dq // 2)), q=np.zeros((B, F)))
    rc = lib().pkm_oracle_backward_full(B, d, H, dq, n, k, v, dt, eps, int(bool(bn_training)),
                                        _ptr(x), _ptr(W),
                                        _ptr(mean), _ptr(var), _ptr(gamma), _ptr(beta), _ptr(C),
                                        _ptr(V), _ptr(indices), _ptr(weights), _ptr(G),
                                        _ptr(out["x"]), _ptr(out["W_q"]), _ptr(out["gamma"]),
                                        _ptr(out["beta"]), _ptr(out["subkeys"]), _ptr(out["q"]))
    if rc != 0:
        raise ValueError("pkm_oracle_backward_full rejected the sizes")
    return out
