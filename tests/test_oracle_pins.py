"""Pins for the fp64 oracle: each check comes from outside the oracle itself.

* brute force over all n^2 explicit keys ("Product Keys Give Transformers
  Million-Slot Memory Layers": "Implied keys vs stored sub-keys" defines key (i, j)
  as left sub-key i joined with right sub-key j; "Search cost: flat vs product
  keys" names the flat search over N = n^2 keys). The product search must return
  the same slots ("Why top-k of each half is enough": exact for Cartesian keys).
* a hand-worked 3x3 example (tests/golden/toy_3x3.json).
* library routines: torch matmul and batch_norm (eval mode) in fp64, torch sort,
  torch index_add.
* closed forms: all-equal sub-keys (every key ties, so the k lowest slots win),
  BN identity, k = 1, softmax sums to one, identity value table.
* central finite differences for the backward; its invariants.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _layer(w, seed=None):
    return synth.make_layer(w, seed=seed)


def _explicit_keys(subkeys, h, n):
    """All n*n keys C[i] (+) C'[j] as an [n*n][dq] fp64 matrix, slot i*n + j."""
    C = subkeys[h, 0].double()
    Cp = subkeys[h, 1].double()
    left = C.repeat_interleave(n, dim=0)      # row i*n+j -> C[i]
    right = Cp.repeat(n, 1)                   # row i*n+j -> C'[j]
    return torch.cat([left, right], dim=1)


# ----------------------------------------------------------------- search pins


@pytest.mark.parametrize("shape", [
    dict(H=1, dq=16, n=16, k=4, d=32, dtype="f32"),     # the tiny workload shape
    dict(H=2, dq=8, n=7, k=3, d=12, dtype="f32"),
    dict(H=3, dq=6, n=5, k=5, d=9, dtype="f32"),        # k = n: every pair is a candidate
    dict(H=1, dq=4, n=9, k=1, d=5, dtype="f32"),        # k = 1
    dict(H=2, dq=10, n=12, k=8, d=16, dtype="bf16"),
    dict(H=2, dq=32, n=24, k=16, d=40, dtype="bf16"),
])
def test_product_topk_equals_flat_bruteforce(shape):
    w = synth.WORKLOADS["tiny"].with_(B=37, d_model=shape["d"], H=shape["H"], dq=shape["dq"],
                                      n=shape["n"], k=shape["k"], v=8, dtype=shape["dtype"],
                                      bn_random=True)
    L = _layer(w, seed=1234 + shape["n"])
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_q=True, want_half=True)
    fi, fs = oracle.flat_topk(r["q"], L["subkeys"], w.H, w.dq, w.n, w.k)
    np.testing.assert_array_equal(r["indices"], fi)
    np.testing.assert_allclose(r["scores"], fs, rtol=1e-12, atol=1e-12)
    # score(i, j) = s1[i] + s2[j] = <q, C[i] (+) C'[j]> for every key, not only the kept ones.
    q = torch.from_numpy(r["q"])
    for h in range(w.H):
        K = _explicit_keys(L["subkeys"], h, w.n)
        full = q[:, h * w.dq:(h + 1) * w.dq] @ K.T                # [B][n*n]
        half = torch.from_numpy(r["half"][:, h])                  # [B][2][n]
        summed = (half[:, 0, :, None] + half[:, 1, None, :]).reshape(w.B, -1)
        torch.testing.assert_close(summed, full, rtol=1e-12, atol=1e-12)


def test_flat_bruteforce_matches_torch_sort():
    """The brute force itself against a library sort of the explicit key scores."""
    w = synth.WORKLOADS["tiny"].with_(B=9, H=2, n=6, k=5, dq=8, d_model=10)
    L = _layer(w, seed=77)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_q=True)
    fi, fs = oracle.flat_topk(r["q"], L["subkeys"], w.H, w.dq, w.n, w.k)
    q = torch.from_numpy(r["q"])
    for h in range(w.H):
        sc = q[:, h * w.dq:(h + 1) * w.dq] @ _explicit_keys(L["subkeys"], h, w.n).T
        for t in range(w.B):
            # lexicographic (score desc, slot asc) via numpy lexsort on (slot, -score)
            order = np.lexsort((np.arange(w.n * w.n), -sc[t].numpy()))[: w.k]
            np.testing.assert_array_equal(fi[t, h], order)
            np.testing.assert_allclose(fs[t, h], sc[t].numpy()[order], rtol=1e-13)


@pytest.mark.slow
def test_product_equals_flat_at_paper_shape_sampled():
    """n = 512 (262,144 slots), H = 4, k = 32, dq = 512 on two sampled tokens."""
    w = synth.WORKLOADS["c512"].with_(B=2)
    L = _layer(w, seed=99)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_q=True, want_out=False)
    fi, fs = oracle.flat_topk(r["q"], L["subkeys"], w.H, w.dq, w.n, w.k)
    np.testing.assert_array_equal(r["indices"], fi)
    np.testing.assert_allclose(r["scores"], fs, rtol=1e-12)


def test_toy_3x3_golden():
    g = json.load(open(os.path.join(GOLDEN, "toy_3x3.json")))
    c = g["layer"]
    n, v = c["n"], c["v"]
    sub = torch.tensor([[c["C_left"], c["C_right"]]], dtype=torch.float32)
    L = dict(x=torch.tensor(c["x"], dtype=torch.float32),
             W_q=torch.tensor(c["W_q"], dtype=torch.float32),
             bn_mean=torch.tensor(c["bn_mean"], dtype=torch.float32),
             bn_var=torch.tensor(c["bn_var"], dtype=torch.float32),
             bn_gamma=torch.tensor(c["bn_gamma"], dtype=torch.float32),
             bn_beta=torch.tensor(c["bn_beta"], dtype=torch.float32),
             subkeys=sub,
             values=torch.tensor([[s, 10 * s] for s in range(n * n)], dtype=torch.float32))
    r = oracle.forward(L, c["H"], c["dq"], n, c["k"], eps=c["bn_eps"], want_half=True)
    e = g["expected"]
    np.testing.assert_array_equal(r["indices"], np.array(e["indices"]))
    np.testing.assert_array_equal(r["scores"], np.array(e["scores"]))
    np.testing.assert_allclose(r["weights"], np.array(e["weights"]), rtol=1e-15)
    np.testing.assert_allclose(r["out"], np.array(e["out"]), rtol=1e-15)
    np.testing.assert_array_equal(r["half"][:, 0, 0], np.array(e["left_scores"]))
    np.testing.assert_array_equal(r["half"][:, 0, 1], np.array(e["right_scores"]))


def test_all_keys_tied_lowest_slots_win():
    """Equal sub-keys in each codebook: all n^2 keys tie; slots 0..k-1 win, uniform w."""
    w = synth.WORKLOADS["tiny"].with_(B=5, H=2, n=8, k=5, dq=6, d_model=7)
    L = _layer(w, seed=5)
    L["subkeys"][:] = L["subkeys"][:, :, :1, :]       # every row = row 0 of its codebook
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    np.testing.assert_array_equal(r["indices"], np.broadcast_to(np.arange(w.k), r["indices"].shape))
    np.testing.assert_allclose(r["weights"], 1.0 / w.k, rtol=1e-14)


def test_duplicate_subkeys_lower_slot_wins():
    """Exact integer arithmetic (eps = 0, BN identity) with duplicated sub-key rows.

    Rows 2 and 5 of C equal row 0, row 3 of C' equals row 1: scores tie exactly and
    the kept slot order must follow (score desc, slot asc), as the brute force does.
    """
    w = synth.WORKLOADS["tiny"].with_(B=16, H=1, n=7, k=6, dq=4, d_model=4, bn_random=False)
    g = torch.Generator().manual_seed(3)
    L = _layer(w, seed=3)
    L["x"] = torch.randint(-3, 4, (w.B, 4), generator=g).float()
    L["W_q"] = torch.eye(4)
    sub = torch.randint(-2, 3, (1, 2, w.n, 2), generator=g).float()
    sub[0, 0, 2] = sub[0, 0, 0]
    sub[0, 0, 5] = sub[0, 0, 0]
    sub[0, 1, 3] = sub[0, 1, 1]
    L["subkeys"] = sub
    r = oracle.forward(L, 1, 4, w.n, w.k, eps=0.0, want_q=True)
    fi, fs = oracle.flat_topk(r["q"], sub, 1, 4, w.n, w.k)
    np.testing.assert_array_equal(r["indices"], fi)
    # Independent library check: lexsort of all 49 exact integer scores.
    q = torch.from_numpy(r["q"])
    sc = (q @ _explicit_keys(sub, 0, w.n).T).numpy()
    for t in range(w.B):
        order = np.lexsort((np.arange(w.n * w.n), -sc[t]))[: w.k]
        np.testing.assert_array_equal(r["indices"][t, 0], order)
    assert (np.diff(r["scores"][..., :], axis=-1) <= 0).all()


# ------------------------------------------------------------ query / BN pins


def test_query_bn_matches_torch_eval_batchnorm():
    w = synth.WORKLOADS["c512"].with_(B=6, d_model=48, H=2, dq=16, n=8, k=4, v=8)
    L = _layer(w, seed=11)
    L["bn_gamma"] = torch.rand(w.H * w.dq) + 0.5
    L["bn_beta"] = torch.randn(w.H * w.dq)
    eps = 1e-5
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, eps=eps, want_q=True, want_half=True)
    acc = L["x"].double() @ L["W_q"].double().T
    ref = torch.nn.functional.batch_norm(acc, L["bn_mean"].double(), L["bn_var"].double(),
                                         L["bn_gamma"].double(), L["bn_beta"].double(),
                                         training=False, eps=eps)
    torch.testing.assert_close(torch.from_numpy(r["q"]), ref, rtol=1e-12, atol=1e-12)
    # Step 3 on its own: each half against its codebook, by library matmul.
    q = ref.view(w.B, w.H, 2, w.dq // 2)
    for h in range(w.H):
        for s in range(2):
            torch.testing.assert_close(torch.from_numpy(r["half"][:, h, s]),
                                       q[:, h, s] @ L["subkeys"][h, s].double().T,
                                       rtol=1e-12, atol=1e-12)


def test_bn_identity_closed_form():
    w = synth.WORKLOADS["tiny"].with_(B=4)
    L = _layer(w, seed=2)
    eps = 1e-5
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, eps=eps, want_q=True)
    acc = (L["x"].double() @ L["W_q"].double().T).numpy()
    np.testing.assert_allclose(r["q"], acc / math.sqrt(1.0 + eps), rtol=1e-14, atol=1e-15)


# ------------------------------------------------------ weights / values pins


def test_softmax_sums_to_one_and_orders_scores():
    w = synth.WORKLOADS["tiny"]
    L = _layer(w)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    np.testing.assert_allclose(r["weights"].sum(-1), 1.0, rtol=1e-14)
    assert (np.diff(r["scores"], axis=-1) <= 0).all()
    assert (np.diff(r["weights"], axis=-1) <= 1e-15).all()
    e = np.exp(r["scores"] - r["scores"][..., :1])
    np.testing.assert_allclose(r["weights"], e / e.sum(-1, keepdims=True), rtol=1e-14)


def test_k1_returns_one_row_per_head():
    w = synth.WORKLOADS["tiny"].with_(B=8, H=3, k=1, dq=8, d_model=12)
    L = _layer(w, seed=4)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    np.testing.assert_array_equal(r["weights"], 1.0)
    V = L["values"].double().numpy()
    np.testing.assert_allclose(r["out"], V[r["indices"][:, :, 0]].sum(1), rtol=1e-14)


def test_identity_value_table_scatters_weights():
    """v = n^2 and V = I: out[t][slot] = sum over heads of that slot's weight."""
    w = synth.WORKLOADS["tiny"].with_(B=10, H=2, n=6, k=4, dq=8, d_model=10, v=36)
    L = _layer(w, seed=8)
    L["values"] = torch.eye(36)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    expect = np.zeros((w.B, 36))
    for t in range(w.B):
        for h in range(w.H):
            for j in range(w.k):
                expect[t, r["indices"][t, h, j]] += r["weights"][t, h, j]
    np.testing.assert_allclose(r["out"], expect, rtol=1e-14, atol=1e-15)


def test_finish_reproduces_forward():
    w = synth.WORKLOADS["tiny"]
    L = _layer(w)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    wt, out = oracle.finish(r["scores"], r["indices"], L["values"])
    np.testing.assert_allclose(wt, r["weights"], rtol=1e-15)
    np.testing.assert_allclose(out, r["out"], rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------ backward pins


def test_backward_grad_scores_finite_differences():
    """L = <grad_out, out>; dL/d(kept score) by central differences in fp64."""
    w = synth.WORKLOADS["tiny"].with_(B=6, H=2, dq=8, d_model=12)
    L = _layer(w, seed=21)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(5))
    _, gs = oracle.backward(L["values"], g, r["indices"], r["weights"])
    G = g.double().numpy()
    h = 1e-6
    fd = np.zeros_like(gs)
    for t in range(w.B):
        for hh in range(w.H):
            for j in range(w.k):
                sp = r["scores"].copy()
                sm = r["scores"].copy()
                sp[t, hh, j] += h
                sm[t, hh, j] -= h
                _, op = oracle.finish(sp, r["indices"], L["values"])
                _, om = oracle.finish(sm, r["indices"], L["values"])
                fd[t, hh, j] = ((op * G).sum() - (om * G).sum()) / (2 * h)
    np.testing.assert_allclose(gs, fd, rtol=1e-6, atol=1e-9)


def test_backward_value_grad_finite_differences():
    """dL/dV[slot] = sum of w * grad_out over the picks of that slot (out is linear in V)."""
    w = synth.WORKLOADS["tiny"].with_(B=5, H=2, dq=8, d_model=12, n=4, k=3, v=6)
    L = _layer(w, seed=22)
    L["values"] = torch.round(L["values"] * 64) / 64   # dyadic, so V +- 0.5 is exact in fp32
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(6))
    gv, _ = oracle.backward(L["values"], g, r["indices"], r["weights"])
    G = g.double().numpy()
    V0 = L["values"].clone()
    fd = np.zeros_like(gv)
    step = 0.5   # out is exactly linear in V, so a large step is exact up to rounding
    for s in range(w.n * w.n):
        for c in range(w.v):
            Vp = V0.clone(); Vp[s, c] += step
            Vm = V0.clone(); Vm[s, c] -= step
            _, op = oracle.finish(r["scores"], r["indices"], Vp)
            _, om = oracle.finish(r["scores"], r["indices"], Vm)
            fd[s, c] = ((op * G).sum() - (om * G).sum()) / (2 * step)
    np.testing.assert_allclose(gv, fd, rtol=1e-9, atol=1e-12)


def test_backward_invariants_and_index_add():
    w = synth.WORKLOADS["tiny"].with_(B=40, H=3, dq=8, d_model=12, v=16)
    L = _layer(w, seed=23)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(7))
    gv, gs = oracle.backward(L["values"], g, r["indices"], r["weights"])
    np.testing.assert_allclose(gs.sum(-1), 0.0, atol=1e-13)
    np.testing.assert_allclose(gv.sum(0), w.H * g.double().sum(0).numpy(), rtol=1e-12, atol=1e-12)
    ref = torch.zeros(w.n * w.n, w.v, dtype=torch.float64)
    contrib = torch.from_numpy(r["weights"]).reshape(-1, 1) * \
        g.double().repeat_interleave(w.H * w.k, dim=0)
    ref.index_add_(0, torch.from_numpy(r["indices"]).reshape(-1).long(), contrib)
    torch.testing.assert_close(torch.from_numpy(gv), ref, rtol=1e-12, atol=1e-13)


def test_backward_row_slot_compaction_matches_dense():
    w = synth.WORKLOADS["tiny"].with_(B=20, H=2, dq=8, d_model=12, v=8)
    L = _layer(w, seed=24)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(8))
    dense, gs = oracle.backward(L["values"], g, r["indices"], r["weights"])
    rows = np.unique(r["indices"])
    slot = -np.ones(w.n * w.n, np.int64)
    slot[rows] = np.arange(rows.size)
    comp, gs2 = oracle.backward(L["values"], g, r["indices"], r["weights"], row_slot=slot,
                                rows=rows.size)
    np.testing.assert_array_equal(comp, dense[rows])
    np.testing.assert_array_equal(gs, gs2)
    untouched = np.setdiff1d(np.arange(w.n * w.n), rows)
    assert not dense[untouched].any()


# ------------------------------------------------------- slot-usage pins


def test_slot_usage_matches_numpy_unique():
    g = torch.Generator().manual_seed(31)
    for slots, picks in ((16, 5), (256, 1000), (262144, 200000)):
        idx = torch.randint(0, slots, (picks,), generator=g).numpy().astype(np.int32)
        n, bad = oracle.slot_usage(idx, slots)
        assert n == np.unique(idx).size and bad == 0


def test_slot_usage_closed_forms():
    assert oracle.slot_usage(np.arange(100, dtype=np.int32), 100) == (100, 0)      # all slots once
    assert oracle.slot_usage(np.full(50, 7, np.int32), 100) == (1, 0)               # one slot
    assert oracle.slot_usage(np.array([3, -1, 100, 3, 99], np.int32), 100) == (2, 2)  # bad ids
    assert oracle.slot_usage(np.zeros(0, np.int32), 10) == (0, 0)


# ------------------------------------------------------- full backward pins


def _loss_and_picks(L, w, G):
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    return float((r["out"] * G).sum()), r["indices"]


@pytest.mark.parametrize("param", ["x", "W_q", "bn_gamma", "bn_beta", "subkeys"])
def test_backward_full_matches_finite_differences(param):
    """dL/dparam of L = <grad_out, out> by central differences through the forward,
    with the picks held fixed (perturbations that change the picks are skipped)."""
    w = synth.WORKLOADS["tiny"].with_(B=6, H=2, dq=8, d_model=10, n=6, k=3, v=8,
                                      bn_random=True)
    L = synth.make_layer(w, seed=41)
    L["bn_gamma"] = torch.rand(w.H * w.dq, generator=torch.Generator().manual_seed(1)) + 0.5
    L["bn_beta"] = torch.randn(w.H * w.dq, generator=torch.Generator().manual_seed(2))
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(3))
    G = g.double().numpy()
    r = oracle.forward(L, w.H, w.dq, w.n, w.k)
    grads = oracle.backward_full(L, r["indices"], r["weights"], g, w.H, w.dq, w.n, w.k)
    key = {"x": "x", "W_q": "W_q", "bn_gamma": "gamma", "bn_beta": "beta",
           "subkeys": "subkeys"}[param]
    base = L[param].clone()
    flat = base.view(-1)
    fd = np.zeros(flat.numel())
    skipped = 0
    h = 2e-4
    for i in range(flat.numel()):
        up, dn = flat.clone(), flat.clone()
        up[i] = flat[i] + h
        dn[i] = flat[i] - h
        du = float(up[i].double() - flat[i].double())     # exact fp32 steps
        dd = float(flat[i].double() - dn[i].double())
        L[param] = up.view_as(base)
        lu, iu = _loss_and_picks(L, w, G)
        L[param] = dn.view_as(base)
        ld, idn = _loss_and_picks(L, w, G)
        L[param] = base
        if not (np.array_equal(iu, r["indices"]) and np.array_equal(idn, r["indices"])):
            fd[i] = np.nan
            skipped += 1
            continue
        fd[i] = (lu - ld) / (du + dd)
    got = grads[key].reshape(-1)
    ok = ~np.isnan(fd)
    assert skipped <= max(2, 0.1 * flat.numel())
    np.testing.assert_allclose(got[ok], fd[ok], rtol=2e-5, atol=1e-7)


def test_backward_full_value_and_score_parts_match_backward():
    """The shared parts: dL/dq summed over a head's sub-keys equals the scores' chain."""
    w = synth.WORKLOADS["tiny"].with_(B=9, H=2, dq=8, d_model=10, n=6, k=3, v=8)
    L = synth.make_layer(w, seed=42)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_q=True)
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(4))
    grads = oracle.backward_full(L, r["indices"], r["weights"], g, w.H, w.dq, w.n, w.k)
    _, gs = oracle.backward(L["values"], g, r["indices"], r["weights"])
    # dL/d(kept score) pushed into q1 through <q1, C[i]>: sum_e dL/dq1[e] * q1[e]
    # equals sum_j g_s[j] * s1[i_j] (Euler: s1 is linear in q1); the same for q2.
    q = r["q"].reshape(w.B, w.H, 2, w.dq // 2)
    gq = grads["q"].reshape(w.B, w.H, 2, w.dq // 2)
    C = L["subkeys"].double().numpy()
    for t in range(w.B):
        for hh in range(w.H):
            for side in range(2):
                sub = r["indices"][t, hh] // w.n if side == 0 else r["indices"][t, hh] % w.n
                s_half = C[hh, side][sub] @ q[t, hh, side]
                np.testing.assert_allclose((gq[t, hh, side] * q[t, hh, side]).sum(),
                                           (gs[t, hh] * s_half).sum(), rtol=1e-10, atol=1e-12)


# ------------------------------------------------------- BatchNorm training-mode pins


def _train_layer(seed=51, **kw):
    shape = dict(B=7, H=2, dq=8, d_model=10, n=6, k=3, v=8, bn_random=True)
    shape.update(kw)
    w = synth.WORKLOADS["tiny"].with_(**shape)
    L = synth.make_layer(w, seed=seed)
    L["bn_gamma"] = torch.rand(w.H * w.dq, generator=torch.Generator().manual_seed(seed + 1)) + 0.5
    L["bn_beta"] = torch.randn(w.H * w.dq, generator=torch.Generator().manual_seed(seed + 2))
    return w, L


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_forward_train_batchnorm_matches_torch(dtype):
    """q, the batch statistics and the running-statistics update against
    torch.nn.functional.batch_norm(training=True) on a library fp64 matmul."""
    w, L = _train_layer(B=13, d_model=24)
    for key in ("x", "W_q", "subkeys", "values"):
        L[key] = L[key].to(dtype)
    mom = 0.3
    r = oracle.forward_train(L, w.H, w.dq, w.n, w.k, eps=1e-5, momentum=mom, want_q=True)
    acc = L["x"].double() @ L["W_q"].double().T
    rm, rv = L["bn_mean"].double().clone(), L["bn_var"].double().clone()
    q = torch.nn.functional.batch_norm(acc, rm, rv, L["bn_gamma"].double(), L["bn_beta"].double(),
                                       training=True, momentum=mom, eps=1e-5)
    np.testing.assert_allclose(r["q"], q.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["batch_mean"], acc.mean(0).numpy(), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(r["batch_var"], acc.var(0, unbiased=False).numpy(), rtol=1e-10)
    np.testing.assert_allclose(r["running_mean"], rm.numpy(), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(r["running_var"], rv.numpy(), rtol=1e-10)


def test_forward_train_search_is_the_flat_top_k_of_its_query():
    """Steps 2-7 on the training-mode query: the picks are the brute-force top-k over
    all n^2 explicit keys of that query."""
    w, L = _train_layer(B=11, n=7, k=4)
    r = oracle.forward_train(L, w.H, w.dq, w.n, w.k, want_q=True)
    idx, sc = oracle.flat_topk(r["q"], L["subkeys"], w.H, w.dq, w.n, w.k)
    np.testing.assert_array_equal(r["indices"], idx)
    np.testing.assert_allclose(r["scores"], sc, rtol=1e-12, atol=1e-12)


def test_forward_train_rejects_one_token():
    w, L = _train_layer(B=1)
    with pytest.raises(ValueError):
        oracle.forward_train(L, w.H, w.dq, w.n, w.k)


@pytest.mark.parametrize("param", ["x", "W_q", "bn_gamma", "bn_beta", "subkeys"])
def test_backward_full_training_bn_matches_finite_differences(param):
    """dL/dparam with training-mode BatchNorm: every perturbation moves the batch
    statistics too, so x and W_q see the mean and variance terms; picks held fixed."""
    w, L = _train_layer(seed=61)
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(7))
    G = g.double().numpy()
    r = oracle.forward_train(L, w.H, w.dq, w.n, w.k)
    grads = oracle.backward_full(L, r["indices"], r["weights"], g, w.H, w.dq, w.n, w.k,
                                 bn_training=True)
    key = {"x": "x", "W_q": "W_q", "bn_gamma": "gamma", "bn_beta": "beta",
           "subkeys": "subkeys"}[param]
    base = L[param].clone()
    flat = base.view(-1)
    fd = np.full(flat.numel(), np.nan)
    h = 2e-4
    for i in range(flat.numel()):
        up, dn = flat.clone(), flat.clone()
        up[i] = flat[i] + h
        dn[i] = flat[i] - h
        du = float(up[i].double() - flat[i].double())
        dd = float(flat[i].double() - dn[i].double())
        L[param] = up.view_as(base)
        ru = oracle.forward_train(L, w.H, w.dq, w.n, w.k)
        L[param] = dn.view_as(base)
        rd = oracle.forward_train(L, w.H, w.dq, w.n, w.k)
        L[param] = base
        if np.array_equal(ru["indices"], r["indices"]) and np.array_equal(rd["indices"], r["indices"]):
            fd[i] = ((ru["out"] * G).sum() - (rd["out"] * G).sum()) / (du + dd)
    ok = ~np.isnan(fd)
    assert (~ok).sum() <= max(2, 0.1 * flat.numel())
    np.testing.assert_allclose(grads[key].reshape(-1)[ok], fd[ok], rtol=2e-5, atol=1e-7)


def test_training_bn_gradient_sums_vanish_through_the_mean():
    """With batch statistics, shifting acc[:, f] by one constant for every token leaves
    q unchanged, so sum_t dL/dacc[t, f] = 0 for every feature. With a constant input
    column x[:, 0] = 1 that sum is dL/dW_q[f][0], which must vanish (it does not in
    inference mode, where the mean is a constant)."""
    w, L = _train_layer(seed=71, d_model=10)
    L["x"][:, 0] = 1.0
    g = torch.randn(w.B, w.v, generator=torch.Generator().manual_seed(9))
    r = oracle.forward_train(L, w.H, w.dq, w.n, w.k)
    grads = oracle.backward_full(L, r["indices"], r["weights"], g, w.H, w.dq, w.n, w.k,
                                 bn_training=True)
    scale = np.abs(grads["W_q"]).max()
    np.testing.assert_allclose(grads["W_q"][:, 0], 0.0, atol=1e-12 * max(1.0, scale))
    inf = oracle.backward_full(L, r["indices"], r["weights"], g, w.H, w.dq, w.n, w.k)
    assert np.abs(inf["W_q"][:, 0]).max() > 1e-6 * scale
