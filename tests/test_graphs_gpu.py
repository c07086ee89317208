"""The library's calls inside CUDA graphs: captured once, replayed on new inputs
copied into the captured buffers, they must give what the same calls give eagerly.

Covered: the tensor-core forward, the small-batch forward (cluster launch,
programmatic dependent launch) and the value backward, whose slot grouping and row
sums run on the library's helper stream (forked from and joined back into the
captured stream by events). Every output of these calls is deterministic, so graph
replays and eager calls must agree bit for bit.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _P():
    import product_key_memory_b200 as mod
    return mod


def _layer(B, n=None):
    w = synth.WORKLOADS["c512"].with_(B=B) if n is None else synth.WORKLOADS["c512"].with_(B=B, n=n)
    L = {k: v.cuda() for k, v in synth.make_layer(w).items()}
    return w, L


def _forward_graph(B, subbatches=1):
    P = _P()
    w, L = _layer(B)
    x_static = L["x"].clone()
    out = torch.empty(B, w.v, device="cuda")
    idx = torch.empty(B, w.H, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(B, w.H, w.k, device="cuda")
    shape = P.make_shape(B, w.d_model, w.H, w.dq, w.n, w.k, w.v, torch.bfloat16)
    with P.options(subbatches=subbatches):
        ws = P.alloc_workspace(shape, False, "cuda")

    def call():
        with P.options(subbatches=subbatches):
            P.pkm_forward(x_static, L["W_q"], L["bn_mean"], L["bn_var"], L["bn_gamma"],
                          L["bn_beta"], L["subkeys"], L["values"], k=w.k, out=out,
                          indices=idx, weights=wt, want_scores=False, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()                      # warm-up outside capture (attributes, helper stream)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    results = []
    for seed in (3, 4):
        x_new = torch.randn(B, w.d_model, generator=torch.Generator().manual_seed(seed))
        x_static.copy_(x_new.to(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        graph_res = (out.clone(), idx.clone(), wt.clone())
        call()
        torch.cuda.synchronize()
        results.append((graph_res, (out.clone(), idx.clone(), wt.clone())))
    assert P.pkm_device_status(ws) == 0
    return results


@pytest.mark.parametrize("B", [1024, 8])
def test_forward_replays_match_eager(B):
    """1024 tokens: the tensor-core kernels; 8 tokens: the small-batch kernels."""
    for (go, gi, gw), (eo, ei, ew) in _forward_graph(B):
        assert torch.equal(gi, ei)
        assert torch.equal(gw, ew)
        assert torch.equal(go, eo)


def test_pipelined_forward_replays_match_eager():
    """4096 tokens in two sub-batches: the first sub-batch's gather runs on the helper
    stream while the second is scored on the captured stream."""
    for (go, gi, gw), (eo, ei, ew) in _forward_graph(4096, subbatches=2):
        assert torch.equal(gi, ei)
        assert torch.equal(gw, ew)
        assert torch.equal(go, eo)


def test_value_backward_replays_match_eager():
    P = _P()
    w, L = _layer(512, n=256)
    out, idx, wt, _ = P.pkm_forward(L["x"], L["W_q"], L["bn_mean"], L["bn_var"],
                                    L["bn_gamma"], L["bn_beta"], L["subkeys"], L["values"],
                                    k=w.k)
    gout = synth.make_grad_out(w).cuda()
    gv = torch.zeros(w.n * w.n, w.v, device="cuda")
    gs = torch.empty(idx.shape, device="cuda")
    shape = P.make_shape(w.B, 0, w.H, 0, w.n, w.k, w.v, torch.bfloat16)
    ws = P.alloc_workspace(shape, True, "cuda")

    def call():
        P.pkm_backward_values(L["values"], idx, wt, gout, gv, gs, w.n, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    gv.zero_()
    g.replay()
    torch.cuda.synchronize()
    graph_gv, graph_gs = gv.clone(), gs.clone()
    gv.zero_()
    call()
    torch.cuda.synchronize()
    assert torch.equal(graph_gs, gs)
    assert torch.equal(graph_gv, gv)
    assert P.pkm_device_status(ws) == 0
    assert P.pkm_device_status(ws) == 0
