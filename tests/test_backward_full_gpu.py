"""GPU parity of pkm_backward (the full backward) against the fp64 oracle, through
the C ABI.

Both sides hold the same picks fixed: the device forward's indices and weights
(fp32) go to the oracle as they are, so near-ties in the forward play no part.
Tolerance for every element of every gradient tensor: |got - ref| <= 1e-4 + 2e-3 |ref|
(the stated bar, with no scaling by the tensor's size). Each check prints its worst
error as a fraction of that bar.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import grad_report

pytestmark = pytest.mark.gpu

NAMES = ("x", "W_q", "bn_gamma", "bn_beta", "subkeys", "values", "scores")
ORACLE_KEY = {"x": "x", "W_q": "W_q", "bn_gamma": "gamma", "bn_beta": "beta",
              "subkeys": "subkeys"}


def _P():
    import product_key_memory_b200 as mod
    return mod


def _grad_check(name, got, ref):
    return grad_report(name, got, ref)


def _with_path(path):
    return _P().options(path=path)


def _device_forward_backward(L, w, gout, path="auto", want=NAMES, init_values=None):
    d = {k: v.cuda() for k, v in L.items()}
    G = gout.cuda()
    with _with_path(path):
        out, idx, wt, _ = _P().pkm_forward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"],
                                           d["bn_gamma"], d["bn_beta"], d["subkeys"],
                                           d["values"], k=w.k)
        shapes = {"x": d["x"].shape, "W_q": d["W_q"].shape, "bn_gamma": d["bn_gamma"].shape,
                  "bn_beta": d["bn_beta"].shape, "subkeys": d["subkeys"].shape,
                  "values": d["values"].shape, "scores": idx.shape}
        grads = {}
        for n in want:
            if n == "values" and init_values is not None:
                grads[n] = init_values.cuda().clone()
            elif n == "values":
                grads[n] = torch.zeros(shapes[n], dtype=torch.float32, device="cuda")
            else:
                grads[n] = torch.full(shapes[n], float("nan"), dtype=torch.float32, device="cuda")
        _P().pkm_backward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"],
                          d["bn_beta"], d["subkeys"], d["values"], idx, wt, G, grads)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), wt.cpu().numpy(), {k: v.cpu() for k, v in grads.items()}


def _oracle_full(L, idx, wt, gout, w, chunks=1):
    """oracle.backward_full over the batch; with chunks > 1 the tokens are split and
    the per-token terms summed (every gradient is a sum over tokens)."""
    if chunks == 1:
        return oracle.backward_full(L, idx, wt.astype(np.float64), gout, w.H, w.dq, w.n, w.k)
    B = L["x"].shape[0]
    bounds = np.linspace(0, B, chunks + 1).astype(int)

    def run(i):
        a, b = bounds[i], bounds[i + 1]
        Ls = dict(L)
        Ls["x"] = L["x"][a:b]
        return oracle.backward_full(Ls, idx[a:b], wt[a:b].astype(np.float64), gout[a:b],
                                    w.H, w.dq, w.n, w.k)

    with cf.ThreadPoolExecutor(max_workers=min(chunks, os.cpu_count() or 1)) as ex:
        parts = list(ex.map(run, range(chunks)))
    out = {"x": np.concatenate([p["x"] for p in parts]),
           "q": np.concatenate([p["q"] for p in parts])}
    for key in ("W_q", "gamma", "beta", "subkeys"):
        out[key] = sum(p[key] for p in parts)
    return out


def _value_grads(L, gout, idx, wt):
    """Oracle grad_values on the touched rows only (the dense fp64 table of a 512^2
    memory would not fit), grad_scores, and the touched row ids."""
    rows = np.unique(idx)
    slot = -np.ones(L["values"].shape[0], np.int64)
    slot[rows] = np.arange(rows.size)
    gv, gs = oracle.backward(L["values"], gout, idx, wt.astype(np.float64), row_slot=slot,
                             rows=rows.size)
    return rows, gv, gs


def _compare_all(L, w, idx, wt, gout, grads, ref, init_values=None):
    for n, key in ORACLE_KEY.items():
        if n in grads:
            got = grads[n].numpy()
            _grad_check("grad_" + n, got, ref[key].reshape(got.shape))
    if "values" in grads or "scores" in grads:
        rows, gv, gs = _value_grads(L, gout, idx, wt)
        if "scores" in grads:
            _grad_check("grad_scores", grads["scores"].numpy(), gs)
        if "values" in grads:
            got = grads["values"]
            base = torch.zeros_like(got) if init_values is None else init_values.float()
            r = torch.as_tensor(rows)
            _grad_check("grad_values rows", (got[r] - base[r]).numpy(), gv)
            keep = torch.ones(got.shape[0], dtype=torch.bool)
            keep[r] = False
            assert torch.equal(got[keep], base[keep]), "untouched value rows changed"


def test_tiny_fp32_every_gradient():
    w = synth.WORKLOADS["tiny"].with_tokens(64)
    L = synth.make_layer(w)
    gout = synth.make_grad_out(w)
    idx, wt, g = _device_forward_backward(L, w, gout)
    _compare_all(L, w, idx, wt, gout, g, _oracle_full(L, idx, wt, gout, w))


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_bf16_ragged_batch_both_query_paths(path):
    """c512 layer shape with 256^2 slots and a batch that leaves ragged tiles."""
    w = synth.WORKLOADS["c512"].with_(B=333, n=256)
    L = synth.make_layer(w)
    gout = synth.make_grad_out(w)
    idx, wt, g = _device_forward_backward(L, w, gout, path=path)
    _compare_all(L, w, idx, wt, gout, g, _oracle_full(L, idx, wt, gout, w, chunks=4))


def test_c512_full_batch():
    """The backward workload: 512^2 slots, B = 4096 tokens, every gradient tensor but
    grad_values checked in full (the oracle's token sum split over threads)."""
    w = synth.WORKLOADS["c512"]
    L = synth.make_layer(w)
    gout = synth.make_grad_out(w)
    want = tuple(n for n in NAMES if n != "values")   # value rows: test_backward_gpu.py
    idx, wt, g = _device_forward_backward(L, w, gout, want=want)
    _compare_all(L, w, idx, wt, gout, g, _oracle_full(L, idx, wt, gout, w, chunks=16))


def test_partial_requests_leave_the_rest_alone():
    """Only grad_subkeys and grad_values requested; grad_values accumulates onto the
    caller's table."""
    w = synth.WORKLOADS["c512"].with_(B=200, n=128)
    L = synth.make_layer(w)
    gout = synth.make_grad_out(w)
    init = torch.randn(w.n * w.n, w.v, generator=torch.Generator().manual_seed(5))
    idx, wt, g = _device_forward_backward(L, w, gout, want=("subkeys", "values"),
                                          init_values=init)
    assert set(g) == {"subkeys", "values"}
    _compare_all(L, w, idx, wt, gout, g, _oracle_full(L, idx, wt, gout, w), init_values=init)


def test_matches_value_backward_bit_for_bit():
    """grad_scores and grad_values come from the same kernels as pkm_backward_values,
    whose sums run in a fixed order: both equal bit for bit."""
    w = synth.WORKLOADS["c512"].with_(B=300, n=256)
    L = synth.make_layer(w)
    gout = synth.make_grad_out(w)
    idx, wt, g = _device_forward_backward(L, w, gout, want=("values", "scores"))
    gv = torch.zeros(w.n * w.n, w.v, device="cuda")
    gs = torch.empty(idx.shape, device="cuda")
    _P().pkm_backward_values(L["values"].cuda(), torch.as_tensor(idx).cuda(),
                             torch.as_tensor(wt).cuda(), gout.cuda(), gv, gs, w.n)
    torch.cuda.synchronize()
    assert torch.equal(gs.cpu(), g["scores"])
    assert torch.equal(gv.cpu(), g["values"])


def test_tied_left_sub_keys():
    """Every left sub-key equal: all left scores tie, so each token's picks are
    (i, j*) for i = 0..k-1. The left rows each get one pick per token, the right row
    j* gets all k of them: long and short sub-key groups side by side."""
    w = synth.WORKLOADS["c512"].with_(B=64, n=128)
    L = synth.make_layer(w)
    L["subkeys"][:, 0] = L["subkeys"][:, 0, :1]
    gout = synth.make_grad_out(w)
    idx, wt, g = _device_forward_backward(L, w, gout, want=("subkeys", "x"))
    ref = _oracle_full(L, idx, wt, gout, w)
    _grad_check("grad_subkeys", g["subkeys"].numpy(), ref["subkeys"].reshape(g["subkeys"].shape))
    _grad_check("grad_x", g["x"].numpy(), ref["x"])


def test_zero_tokens():
    w = synth.WORKLOADS["tiny"].with_(B=0)
    L = synth.make_layer(w)
    d = {k: v.cuda() for k, v in L.items()}
    idx = torch.empty(0, w.H, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(0, w.H, w.k, device="cuda")
    gW = torch.full(d["W_q"].shape, 3.0, device="cuda")
    _P().pkm_backward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"], d["bn_beta"],
                      d["subkeys"], d["values"], idx, wt,
                      torch.empty(0, w.v, device="cuda"), {"W_q": gW})
    torch.cuda.synchronize()
    # a sum over no tokens: the requested parameter gradients are zero
    assert torch.all(gW == 0.0)


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_wide_layer_ragged_gemm_tiles(path):
    """d_model 1600, H = 8, v = 1600: the GEMMs' N = 1600 leaves a ragged 256-column
    tile, K = 200 tokens a ragged 64-row block, and the small output splits K."""
    w = synth.WORKLOADS["wide"].with_(B=200, n=256)
    L = synth.make_layer(w)
    gout = synth.make_grad_out(w)
    idx, wt, g = _device_forward_backward(L, w, gout, path=path,
                                          want=("x", "W_q", "bn_gamma", "bn_beta", "subkeys"))
    _compare_all(L, w, idx, wt, gout, g, _oracle_full(L, idx, wt, gout, w, chunks=4))
