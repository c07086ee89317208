"""Stage tracing (pkm_trace_enable / pkm_trace_read) on the GPU: per-stage CUDA-event
times of the forward (one event per stage boundary on the caller's stream) and of the
value backward (whose slot grouping runs on the library's helper stream).

Each traced call must report every stage it ran with a positive time, the call's own
span must cover its stages (they run in order on one stream, so their sum is at most
the call's time), and the launch counts must match the kernels the call issued.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _P():
    import product_key_memory_b200 as mod
    return mod


def _layer(name, B):
    w = synth.WORKLOADS[name].with_(B=B)
    return w, {k: v.cuda() for k, v in synth.make_layer(w).items()}


def _forward(P, w, d, ws=None):
    return P.pkm_forward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"],
                         d["bn_beta"], d["subkeys"], d["values"], k=w.k, workspace=ws)


@pytest.mark.parametrize("name,B,path,stages,launches", [
    ("c512", 1024, "auto", (0, 1, 2), 3),      # tensor-core kernels
    ("c512", 4, "auto", (2,), 3),              # small batch, three kernels (decode mode)
    ("c512", 16, "auto", (2,), 3),             # small batch, three kernels (MMA tiles)
    ("c512", 16, "small_fused", (2,), 1),      # small batch, one cooperative kernel
    ("tiny", 64, "simt", (0, 1, 2), 3),        # CUDA-core kernels (fp32)
    ("tiny", 112, "auto", (2,), 3),            # fp32 small batch: CUDA-core kernels
    ("tiny", 113, "auto", (0, 1, 2), 3),       # ... up to 112 tokens
    # The automatic cut-off depends on the heads: H = 8 takes the small-batch kernels
    # up to 240 tokens, the tensor-core kernels above; H = 4 up to 384. A pinned form
    # takes them to 512.
    ("wide", 240, "auto", (2,), 3),
    ("wide", 241, "auto", (0, 1, 2), 3),
    ("wide", 256, "small_split", (2,), 3),
    ("c1024", 384, "auto", (2,), 3),
    ("c1024", 385, "auto", (0, 1, 2), 3),
])
def test_forward_stages(name, B, path, stages, launches):
    P = _P()
    w, d = _layer(name, B)
    with P.options(path=path):
        _forward(P, w, d)  # warm-up (kernel attributes)
        torch.cuda.synchronize()
        P.pkm_trace_read(0)
        P.pkm_trace_enable(True)
        try:
            n = 3
            for _ in range(n):
                _forward(P, w, d)
            ms, calls, nl = P.pkm_trace_read(0)
        finally:
            P.pkm_trace_enable(False)
    assert calls == n
    assert nl == n * launches
    for st in range(3):
        assert (ms[st] > 0) == (st in stages), ms
    assert ms[3] > 0
    assert sum(ms[:3]) <= ms[3] * (1 + 1e-6) + 1e-6


def test_pipelined_forward_stages():
    """Two sub-batches: the gathers on the helper stream, the call's span closed on the
    caller's stream after it waits for them."""
    P = _P()
    w, d = _layer("c512", 4096)
    with P.options(subbatches=2):
        _forward(P, w, d)
        torch.cuda.synchronize()
        P.pkm_trace_read(0)
        P.pkm_trace_enable(True)
        try:
            _forward(P, w, d)
            ms, calls, nl = P.pkm_trace_read(0)
        finally:
            P.pkm_trace_enable(False)
    assert calls == 1 and nl == 6
    assert all(m > 0 for m in ms), ms
    # The last gather ends before the call's span does.
    assert ms[3] >= ms[2] / 2


def test_value_backward_stages():
    P = _P()
    w, d = _layer("c512", 512)
    out, idx, wt, _ = _forward(P, w, d)
    gout = torch.randn(w.B, w.v, device="cuda").to(torch.bfloat16)
    gv = torch.zeros(w.n * w.n, w.v, device="cuda")
    gs = torch.empty(idx.shape, device="cuda")
    P.pkm_backward_values(d["values"], idx, wt, gout, gv, gs, w.n)
    torch.cuda.synchronize()
    P.pkm_trace_read(1)
    P.pkm_trace_enable(True)
    try:
        P.pkm_backward_values(d["values"], idx, wt, gout, gv, gs, w.n)
        ms, calls, _ = P.pkm_trace_read(1)
    finally:
        P.pkm_trace_enable(False)
    assert calls == 1
    assert ms[0] > 0 and ms[1] > 0 and ms[3] > 0
    # Both parts are inside the call's span: it ends after the helper stream's work.
    assert ms[3] >= max(ms[0], ms[1]) * (1 - 1e-6)
