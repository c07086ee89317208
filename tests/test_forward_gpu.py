"""GPU parity of pkm_forward against the fp64 oracle (called through the C ABI).

Tolerances (tests/parity.py): indices bit-exact except fp64 near-ties within 1e-5
relative of the oracle's k-th score (counted, at most 1% of (token, head));
weights, kept scores and out within 1e-4 absolute + 2e-3 relative.
"""
import functools
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import compare_forward, to_numpy

pytestmark = pytest.mark.gpu

P = None


def _lib():
    global P
    if P is None:
        import product_key_memory_b200 as mod
        P = mod
    return P


@functools.lru_cache(maxsize=2)
def _layer_cached(name, B):
    w = synth.WORKLOADS[name].with_tokens(B)
    return w, synth.make_layer(w)


def _to_dev(L):
    return {k: v.cuda() for k, v in L.items()}


def _gpu_forward(L, w, path="auto"):
    with _lib().options(path=path):
        d = _to_dev(L)
        out, idx, wt, sc = _lib().pkm_forward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"],
                                              d["bn_gamma"], d["bn_beta"], d["subkeys"],
                                              d["values"], k=w.k)
        torch.cuda.synchronize()
        return to_numpy(out, idx, wt, sc)


def _check(L, w, rows=None, path="auto", **kw):
    g = _gpu_forward(L, w, path)
    if rows is not None:
        g = {k: (None if v is None else v[rows]) for k, v in g.items()}
        Ls = dict(L)
        Ls["x"] = L["x"][torch.as_tensor(rows)]
    else:
        Ls = L
    r = oracle.forward(Ls, w.H, w.dq, w.n, w.k, want_half=True)
    stats = compare_forward(g, r, L["values"], w.n, **kw)
    print(w.name, w.B, path, stats)
    return g, r, stats


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_tiny_all_fp32(path):
    w, L = _layer_cached("tiny", 64)
    _check(L, w, path=path)


@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("name,B", [("c512", 333), ("c1024", 301), ("wide", 203)])
def test_bf16_shapes_ragged_batch(name, B, path):
    """Paper shapes with a token count that leaves a ragged last tile."""
    w = synth.WORKLOADS[name].with_tokens(B)
    if name != "c512":
        w = w.with_(n=256)     # the 1024^2 tables are exercised at full size below
    L = synth.make_layer(w)
    _check(L, w, path=path)


def test_c512_full_batch():
    """512^2 slots, B = 4096 tokens, every token checked."""
    w, L = _layer_cached("c512", 4096)
    _check(L, w)


def test_c1024_full_batch():
    """1024^2 slots, B = 16384 tokens (the benchmark launch), every token checked."""
    w, L = _layer_cached("c1024", 16384)
    _check(L, w)


def test_wide_full_batch_sampled():
    """d_model 1600, H = 8, 1024^2 slots, v = 1600, B = 16384; every 8th token checked."""
    w, L = _layer_cached("wide", 16384)
    rows = np.arange(0, w.B, 8)
    _check(L, w, rows=rows)


@pytest.mark.parametrize("k", [1, 3, 16, 32])
def test_k_values(k):
    w = synth.WORKLOADS["c512"].with_(B=97, n=256, k=k)
    L = synth.make_layer(w)
    _check(L, w)


def test_k_equals_n_small_codebooks():
    w = synth.WORKLOADS["tiny"].with_(B=50, n=8, k=8, dq=16, d_model=24, v=16)
    L = synth.make_layer(w)
    _check(L, w)


def test_one_token():
    w = synth.WORKLOADS["c512"].with_(B=1, n=256)
    L = synth.make_layer(w)
    _check(L, w)


def test_zero_tokens_launches_nothing():
    w = synth.WORKLOADS["tiny"].with_(B=0)
    L = synth.make_layer(w)
    d = _to_dev(L)
    out = torch.full((0, w.v), 7.0, device="cuda")
    o, i, wt, s = _lib().pkm_forward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"],
                                     d["bn_beta"], d["subkeys"], d["values"], k=w.k, out=out)
    torch.cuda.synchronize()
    assert o.shape == (0, w.v) and i.shape == (0, w.H, w.k)


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_exact_ties_go_to_lower_slot(path):
    """Left codebook of identical rows: every left score ties, so the k best keys are
    (i, j*) for i = 0..k-1 with j* the best right sub-key: slots i*n + j*, equal weights."""
    w = synth.WORKLOADS["c512"].with_(B=64, n=256)
    L = synth.make_layer(w)
    L["subkeys"][:, 0] = L["subkeys"][:, 0, :1]
    g = _gpu_forward(L, w, path)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_half=True)
    jstar = r["half"][:, :, 1].argmax(-1)                     # [B][H]
    expect = np.arange(w.k)[None, None, :] * w.n + jstar[..., None]
    np.testing.assert_array_equal(r["indices"], expect)       # the oracle's own answer
    np.testing.assert_array_equal(g["indices"], expect)
    np.testing.assert_allclose(g["weights"], 1.0 / w.k, rtol=1e-6)


def test_all_keys_tied():
    w = synth.WORKLOADS["c512"].with_(B=40, n=256)
    L = synth.make_layer(w)
    L["subkeys"][:] = L["subkeys"][:, :, :1]
    g = _gpu_forward(L, w)
    np.testing.assert_array_equal(g["indices"], np.broadcast_to(np.arange(w.k), g["indices"].shape))


@pytest.mark.parametrize("name,B,n", [("c512", 1000, 512), ("wide", 257, 256)])
def test_tensor_core_and_simt_paths_agree(name, B, n):
    """Both implementations of the query network and per-half search, same inputs:
    identical picks except fp32 near-ties, and outputs within the parity tolerance."""
    w = synth.WORKLOADS[name].with_(B=B, n=n)
    L = synth.make_layer(w)
    a = _gpu_forward(L, w, "auto")
    b = _gpu_forward(L, w, "simt")
    same = (a["indices"] == b["indices"]).all(-1)
    assert same.mean() > 0.99
    ok = same[..., None].repeat(w.k, -1)
    np.testing.assert_allclose(a["weights"][ok], b["weights"][ok], rtol=2e-3, atol=1e-4)
    np.testing.assert_allclose(a["scores"][ok], b["scores"][ok], rtol=2e-3, atol=1e-4)
