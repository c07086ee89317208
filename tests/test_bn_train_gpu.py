"""GPU parity of BatchNorm in training mode (pkm_forward_train, pkm_backward_train)
against the fp64 oracle, through the C ABI.

Forward: picks bit-exact except fp64 near-ties (tests/parity.py); out, weights,
kept scores, batch statistics and the updated running statistics within
1e-4 + 2e-3 |ref|. Backward: every gradient within 2e-3 |ref| + 1e-4 max(1, max|ref|)
(the size-scaled bar of the full-backward tests), on the device forward's picks.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import allclose_report, compare_forward, grad_report, to_numpy

pytestmark = pytest.mark.gpu


def _P():
    import product_key_memory_b200 as mod
    return mod


def _Path(path):
    return _P().options(path=path)


def _layer(name, **kw):
    w = synth.WORKLOADS[name].with_(**kw)
    return w, synth.make_layer(w)


def _device_train_forward(L, w, momentum, path="auto"):
    d = {k: v.cuda() for k, v in L.items()}
    rm, rv = d["bn_mean"].clone(), d["bn_var"].clone()
    with _Path(path):
        out, idx, wt, sc, bm, bv = _P().pkm_forward_train(
            d["x"], d["W_q"], rm, rv, d["bn_gamma"], d["bn_beta"], d["subkeys"], d["values"],
            k=w.k, momentum=momentum)
    torch.cuda.synchronize()
    g = to_numpy(out, idx, wt, sc)
    g.update(batch_mean=bm.cpu().numpy(), batch_var=bv.cpu().numpy(),
             running_mean=rm.cpu().numpy(), running_var=rv.cpu().numpy())
    return g, d, idx, wt, bm, bv


def _check_forward(L, w, momentum=0.1, path="auto"):
    g, d, idx, wt, bm, bv = _device_train_forward(L, w, momentum, path)
    r = oracle.forward_train(L, w.H, w.dq, w.n, w.k, momentum=momentum, want_half=True)
    for key in ("batch_mean", "batch_var", "running_mean", "running_var"):
        allclose_report(key, g[key], r[key])
    stats = compare_forward(g, r, L["values"], w.n)
    print(w.name, w.B, path, stats)
    return g, d, idx, wt, bm, bv


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_forward_train_tiny_and_ragged(path):
    w, L = _layer("tiny", B=64)
    _check_forward(L, w, momentum=0.2, path=path)
    w, L = _layer("c512", B=333, n=256)
    _check_forward(L, w, path=path)


def test_forward_train_c1024_full_batch():
    """1024^2 slots, 16,384 tokens (the benchmark shape), every token checked."""
    w, L = _layer("c1024", B=16384)
    _check_forward(L, w)


def test_running_statistics_momentum_limits():
    w, L = _layer("c512", B=300, n=256)
    g0, *_ = _device_train_forward(L, w, 0.0)
    np.testing.assert_array_equal(g0["running_mean"], L["bn_mean"].numpy())
    np.testing.assert_array_equal(g0["running_var"], L["bn_var"].numpy())
    g1, *_ = _device_train_forward(L, w, 1.0)
    np.testing.assert_allclose(g1["running_mean"], g1["batch_mean"], rtol=0, atol=0)
    np.testing.assert_allclose(g1["running_var"], g1["batch_var"] * w.B / (w.B - 1), rtol=1e-6)


def _grad_check(name, got, ref):
    return grad_report(name, got, ref)


def _check_backward(L, w, path="auto"):
    g, d, idx, wt, bm, bv = _device_train_forward(L, w, 0.1, path)
    gout = synth.make_grad_out(w)
    F = w.H * w.dq
    grads = {"x": torch.empty(w.B, w.d_model, device="cuda"),
             "W_q": torch.empty(F, w.d_model, device="cuda"),
             "bn_gamma": torch.empty(F, device="cuda"), "bn_beta": torch.empty(F, device="cuda"),
             "subkeys": torch.empty(w.H, 2, w.n, w.dq // 2, device="cuda"),
             "scores": torch.empty(idx.shape, device="cuda")}
    with _Path(path):
        _P().pkm_backward(d["x"], d["W_q"], bm, bv, d["bn_gamma"], d["bn_beta"], d["subkeys"],
                          d["values"], idx, wt, gout.cuda(), grads, bn_training=True)
    torch.cuda.synchronize()
    ref = oracle.backward_full(L, g["indices"], g["weights"], gout, w.H, w.dq, w.n, w.k,
                               bn_training=True)
    for n, key in (("x", "x"), ("W_q", "W_q"), ("bn_gamma", "gamma"), ("bn_beta", "beta"),
                   ("subkeys", "subkeys")):
        got = grads[n].cpu().numpy()
        _grad_check("grad_" + n, got, ref[key].reshape(got.shape))
    # dL/dacc sums to zero over tokens under batch statistics; with the bias-free
    # linear map that shows as sum_t dL/dx[t] = (sum_t dL/dacc[t]) W_q = 0.
    gx = grads["x"].double().sum(0).cpu().numpy()
    assert np.abs(gx).max() <= 1e-3 * max(1.0, float(np.abs(ref["x"]).max())) * np.sqrt(w.B)


def test_backward_train_tiny_fp32():
    w, L = _layer("tiny", B=64)
    _check_backward(L, w)


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_backward_train_ragged_both_paths(path):
    w, L = _layer("c512", B=333, n=256)
    _check_backward(L, w, path)


def test_backward_train_c512_full_batch():
    """The backward workload's shape, 4096 tokens, every gradient in full."""
    w, L = _layer("c512", B=4096)
    _check_backward(L, w)
