"""GPU parity of the small-batch forward against the fp64 oracle, through the C ABI, in
both forms: the single cooperative kernel and the three kernels. pkm_forward picks the
three kernels by itself up to 384 tokens with H <= 4 and 240 with more heads on bf16
layers whose query and scores run as tensor-core tiles (112 / 96 otherwise); a pinned
form takes up to 512 tokens for any H <= 8. Up to 8 tokens both forms run in decode
mode, above it (bf16) the query network and the per-half scores are warp-level MMA
tiles of 16 tokens.

Same bar as tests/test_forward_gpu.py: indices bit-exact except fp64 near-ties
within 1e-5 relative of the k-th score; weights, kept scores and out within
1e-4 + 2e-3 |ref|.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import compare_forward, to_numpy

pytestmark = pytest.mark.gpu


def _P():
    import product_key_memory_b200 as mod
    return mod


def _forward(L, w, path=None):
    with _P().options(path=path or "auto"):
        d = {k: v.cuda() for k, v in L.items()}
        out, idx, wt, sc = _P().pkm_forward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"],
                                            d["bn_gamma"], d["bn_beta"], d["subkeys"],
                                            d["values"], k=w.k)
        torch.cuda.synchronize()
        return to_numpy(out, idx, wt, sc)


def _check(L, w, path=None):
    g = _forward(L, w, path)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_half=True)
    stats = compare_forward(g, r, L["values"], w.n)
    print(w.name, w.B, stats)
    return g, r


# The two small-batch forms, each forced: the single cooperative kernel and the three
# kernels ("auto" picks the first up to 32 tokens and the second above).
FORMS = ["small_fused", "small_split"]


@pytest.mark.parametrize("path", FORMS)
@pytest.mark.parametrize("B", [1, 7, 8, 32, 64, 96, 112])
def test_c1024_small_batches(B, path):
    w = synth.WORKLOADS["c1024"].with_(B=B)
    _check(synth.make_layer(w), w, path)


@pytest.mark.parametrize("name,B", [("c1024", 256), ("c1024", 384), ("c512", 376),
                                    ("wide", 240)])
def test_larger_batches_default_choice(name, B):
    """The automatic choice up to its cut-off: the three kernels, MMA tiles over several
    16-token tiles (a ragged last one at 376), and gathers of more (token, head) CTAs
    than the GPU holds at once with the default register budget."""
    w = synth.WORKLOADS[name].with_(B=B)
    _check(synth.make_layer(w), w)


@pytest.mark.parametrize("path", FORMS)
@pytest.mark.parametrize("name,B", [("c512", 33), ("wide", 4), ("wide", 16), ("wide", 112),
                                    ("tiny", 5)])
def test_other_shapes(name, B, path):
    w = synth.WORKLOADS[name].with_(B=B)
    _check(synth.make_layer(w), w, path)


@pytest.mark.parametrize("path", FORMS)
@pytest.mark.parametrize("dq,n,B", [(128, 512, 40), (128, 512, 3), (48, 256, 20)])
def test_query_half_widths(dq, n, B, path):
    """bf16 layers with narrower query halves: dq/2 = 64 takes the MMA tiles (two
    32-wide K-blocks per sub-key row; 3 tokens decode mode), dq/2 = 24 (not a multiple
    of 32) the CUDA-core kernels above decode mode."""
    w = synth.WORKLOADS["c512"].with_(B=B, dq=dq, n=n)
    _check(synth.make_layer(w), w, path)


@pytest.mark.parametrize("path", FORMS)
@pytest.mark.parametrize("B", [3, 9])
@pytest.mark.parametrize("k,n", [(1, 256), (3, 256), (8, 8), (32, 32), (32, 100)])
def test_k_and_small_codebooks(k, n, B, path):
    """3 tokens take the decode mode (a warp per W_q row or per 8 sub-keys, lanes over
    the contraction), 9 tokens the MMA tiles; n = 8, 32, 100 leave the last 64-sub-key
    chunk ragged (sub-keys past n read as zeros and are never picked)."""
    w = synth.WORKLOADS["c512"].with_(B=B, n=n, k=k)
    _check(synth.make_layer(w), w, path)


def test_odd_half_query_goes_to_large_batch_kernels():
    """fp32 with dq = 6 (halves of 3 elements): the small-batch scoring loop takes
    element pairs, so such a layer runs on the large-batch CUDA-core kernels and must
    still match the oracle."""
    w = synth.WORKLOADS["tiny"].with_(B=4, dq=6)
    _check(synth.make_layer(w), w)


@pytest.mark.parametrize("B", [3, 40])
def test_fused_and_three_kernel_forms_agree(B):
    """Same arithmetic in both forms (3 tokens: decode mode; 40: MMA tiles): picks,
    weights and scores bit for bit; out up to the order in which the H*k rows are
    added."""
    w = synth.WORKLOADS["c1024"].with_(B=B)
    L = synth.make_layer(w)
    a = _forward(L, w, "small_fused")
    b = _forward(L, w, "small_split")
    np.testing.assert_array_equal(a["indices"], b["indices"])
    np.testing.assert_array_equal(a["weights"], b["weights"])
    np.testing.assert_array_equal(a["scores"], b["scores"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("path", FORMS)
@pytest.mark.parametrize("B", [2, 12])
def test_exact_ties_go_to_lower_slot(path, B):
    w = synth.WORKLOADS["c512"].with_(B=B, n=256)
    L = synth.make_layer(w)
    L["subkeys"][:, 0] = L["subkeys"][:, 0, :1]
    g = _forward(L, w, path)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_half=True)
    jstar = r["half"][:, :, 1].argmax(-1)
    expect = np.arange(w.k)[None, None, :] * w.n + jstar[..., None]
    np.testing.assert_array_equal(g["indices"], expect)
    np.testing.assert_allclose(g["weights"], 1.0 / w.k, rtol=1e-6)


def test_small_and_tensor_core_paths_agree():
    """The same 48 tokens through the small-batch kernels and the large-batch
    tensor-core kernels: identical picks except fp32 near-ties."""
    w = synth.WORKLOADS["c1024"].with_(B=48)
    L = synth.make_layer(w)
    a = _forward(L, w)
    b = _forward(L, w, "tc")
    same = (a["indices"] == b["indices"]).all(-1)
    assert same.mean() > 0.98
    ok = same[..., None].repeat(w.k, -1)
    np.testing.assert_allclose(a["weights"][ok], b["weights"][ok], rtol=2e-3, atol=1e-4)
    np.testing.assert_allclose(a["out"][same.all(-1)], b["out"][same.all(-1)], rtol=2e-3, atol=1e-4)


def test_forward_train_small_batch():
    """BatchNorm training mode on 8 tokens runs the small-batch forward."""
    w = synth.WORKLOADS["c512"].with_(B=8)
    L = synth.make_layer(w)
    d = {k: v.cuda() for k, v in L.items()}
    rm, rv = d["bn_mean"].clone(), d["bn_var"].clone()
    out, idx, wt, sc, bm, bv = _P().pkm_forward_train(d["x"], d["W_q"], rm, rv, d["bn_gamma"],
                                                      d["bn_beta"], d["subkeys"], d["values"],
                                                      k=w.k)
    torch.cuda.synchronize()
    r = oracle.forward_train(L, w.H, w.dq, w.n, w.k, want_half=True)
    compare_forward(to_numpy(out, idx, wt, sc), r, L["values"], w.n)
    np.testing.assert_allclose(bm.cpu().numpy(), r["batch_mean"], rtol=2e-3, atol=1e-4)
    np.testing.assert_allclose(rv.cpu().numpy(), r["running_var"], rtol=2e-3, atol=1e-4)
