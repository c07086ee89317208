"""GPU parity of pkm_backward_values against the fp64 oracle (through the C ABI).

Both sides get the same indices and weights: the oracle's forward picks, rounded
to fp32 for the device. Tolerance: 1e-4 absolute + 2e-3 relative on grad_scores
and on every touched row of grad_values; untouched rows must stay exactly as the
caller left them. The value gradient sums each slot's picks in a fixed order, so two
runs on the same inputs must agree bit for bit, whatever the group sizes.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import allclose_report

pytestmark = pytest.mark.gpu


def _P():
    import product_key_memory_b200 as mod
    return mod


def _run(values, idx, w, gout, n, init=None):
    dev = "cuda"
    V = values.to(dev)
    I = torch.as_tensor(idx, dtype=torch.int32).to(dev).contiguous()
    W = torch.as_tensor(w, dtype=torch.float32).to(dev).contiguous()
    G = gout.to(dev)
    gv = torch.zeros(values.shape[0], values.shape[1], dtype=torch.float32, device=dev) \
        if init is None else init.to(dev).clone()
    gs = torch.empty(I.shape, dtype=torch.float32, device=dev)
    _P().pkm_backward_values(V, I, W, G, gv, gs, n)
    torch.cuda.synchronize()
    return gv, gs


def _compare(values, idx, w32, gout, gv, gs):
    rows = np.unique(idx)
    slot = -np.ones(values.shape[0], np.int64)
    slot[rows] = np.arange(rows.size)
    ref_gv, ref_gs = oracle.backward(values, gout, idx, w32.astype(np.float64), row_slot=slot,
                                     rows=rows.size)
    allclose_report("grad_scores", gs.cpu().numpy(), ref_gs)
    got_rows = gv[torch.as_tensor(rows, device=gv.device)].cpu().numpy()
    allclose_report("grad_values rows", got_rows, ref_gv)
    mask = torch.ones(values.shape[0], dtype=torch.bool, device=gv.device)
    mask[torch.as_tensor(rows, device=gv.device)] = False
    assert int(torch.count_nonzero(gv[mask])) == 0, "untouched rows were written"
    return rows.size


def test_backward_c512_forward_picks():
    """The backward workload: c512 forward picks, grad_out ~ N(0, 1) bf16 [4096][1024]."""
    w = synth.WORKLOADS["c512"]
    L = synth.make_layer(w)
    r = oracle.forward(L, w.H, w.dq, w.n, w.k, want_out=False)
    w32 = r["weights"].astype(np.float32)
    gout = synth.make_grad_out(w)
    gv, gs = _run(L["values"], r["indices"], w32, gout, w.n)
    u = _compare(L["values"], r["indices"], w32, gout, gv, gs)
    print("unique rows", u, "of", r["indices"].size, "picks")


def test_backward_hot_rows_cross_windows():
    """Skewed picks: every pick from 40 slots, so groups span many 32-pick windows."""
    B, H, k, n, v = 700, 4, 32, 128, 256
    idx, w32 = synth.random_selection(B, H, k, n * n, seed=5, hot_rows=40)
    g = synth.generator(6)
    values = (torch.randn(n * n, v, generator=g) / 16).to(torch.bfloat16)
    gout = torch.randn(B, v, generator=g).to(torch.bfloat16)
    gv, gs = _run(values, idx.numpy(), w32.numpy(), gout, n)
    _compare(values, idx.numpy(), w32.numpy(), gout, gv, gs)


def test_backward_uniform_random_fp32_small():
    B, H, k, n, v = 129, 2, 4, 16, 32
    idx, w32 = synth.random_selection(B, H, k, n * n, seed=9)
    g = synth.generator(10)
    values = torch.randn(n * n, v, generator=g)
    gout = torch.randn(B, v, generator=g)
    gv, gs = _run(values, idx.numpy(), w32.numpy(), gout, n)
    _compare(values, idx.numpy(), w32.numpy(), gout, gv, gs)


def test_backward_accumulates_into_grad_table():
    B, H, k, n, v = 64, 2, 8, 32, 64
    idx, w32 = synth.random_selection(B, H, k, n * n, seed=11)
    g = synth.generator(12)
    values = torch.randn(n * n, v, generator=g).to(torch.bfloat16)
    gout = torch.randn(B, v, generator=g).to(torch.bfloat16)
    init = torch.randn(n * n, v, generator=g)
    gv0, _ = _run(values, idx.numpy(), w32.numpy(), gout, n)
    gv1, _ = _run(values, idx.numpy(), w32.numpy(), gout, n, init=init)
    torch.testing.assert_close(gv1.cpu(), init + gv0.cpu(), rtol=1e-6, atol=1e-6)


def test_backward_bad_slot_is_reported_not_written():
    """A slot id outside [0, n*n) is skipped and reported through the status word."""
    B, H, k, n, v = 16, 1, 4, 8, 32
    idx, w32 = synth.random_selection(B, H, k, n * n, seed=13)
    idx[3, 0, 2] = n * n + 5
    idx[7, 0, 0] = -1
    g = synth.generator(14)
    values = torch.randn(n * n, v, generator=g)
    gout = torch.randn(B, v, generator=g)
    P = _P()
    V, I, W, G = values.cuda(), idx.cuda(), w32.cuda(), gout.cuda()
    gv = torch.zeros(n * n, v, device="cuda")
    gs = torch.empty(B, H, k, device="cuda")
    shape = P.make_shape(B, 0, H, 0, n, k, v, torch.float32)
    ws = P.alloc_workspace(shape, True)
    P.pkm_backward_values(V, I, W, G, gv, gs, n, workspace=ws)
    assert P.pkm_device_status(ws) == -5
    assert P.pkm_device_status(ws) == 0          # cleared by the first read
    good = idx.clone()
    keep = (good >= 0) & (good < n * n)
    ref = torch.zeros(n * n, v, dtype=torch.float64)
    contrib = (w32.double() * keep).reshape(-1, 1) * gout.double().repeat_interleave(H * k, 0)
    ref.index_add_(0, good.clamp(0, n * n - 1).reshape(-1).long(), contrib)
    torch.testing.assert_close(gv.cpu().double(), ref, rtol=2e-3, atol=1e-4)


def _skewed(B, H, k, n, v, hot, seed):
    idx, w32 = synth.random_selection(B, H, k, n * n, seed=seed, hot_rows=hot)
    g = synth.generator(seed + 1)
    values = (torch.randn(n * n, v, generator=g) / 16).to(torch.bfloat16)
    gout = torch.randn(B, v, generator=g).to(torch.bfloat16)
    return values, idx.numpy(), w32.numpy(), gout


@pytest.mark.parametrize("B,hot", [(4096, 40), (600, 64), (300, 2000)])
def test_backward_group_sizes_against_oracle(B, hot):
    """Every pick from `hot` slots: groups of ~13,000 picks (split into work items with
    partial rows), ~1,200 picks (one work item each) and ~19 picks (summed inline)."""
    values, idx, w32, gout = _skewed(B, 4, 32, 256, 256, hot, seed=21 + hot)
    gv, gs = _run(values, idx, w32, gout, 256)
    _compare(values, idx, w32, gout, gv, gs)


@pytest.mark.parametrize("hot", [0, 40])
def test_backward_is_bit_for_bit_repeatable(hot):
    """Two runs on the same inputs (uniform picks, and picks from 40 hot slots on the
    c512 table size) give identical grad_values and grad_scores."""
    if hot:
        values, idx, w32, gout = _skewed(4096, 4, 32, 512, 1024, hot, seed=31)
    else:
        idx_t, w_t = synth.random_selection(4096, 4, 32, 512 * 512, seed=33)
        g = synth.generator(34)
        values = (torch.randn(512 * 512, 1024, generator=g) / 32).to(torch.bfloat16)
        gout = torch.randn(4096, 1024, generator=g).to(torch.bfloat16)
        idx, w32 = idx_t.numpy(), w_t.numpy()
    gv1, gs1 = _run(values, idx, w32, gout, 512)
    gv2, gs2 = _run(values, idx, w32, gout, 512)
    assert torch.equal(gv1, gv2)
    assert torch.equal(gs1, gs2)
