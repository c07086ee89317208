"""pkm_backward_values_noalloc against pkm_backward_values, through the C ABI.

The no-allocation entry point serves callers that cannot allocate device memory
where they run the backward; it keeps its scratch in a fixed array inside the
library. Its results must match the regular entry point's (which uses a caller
workspace) within the parity tolerance, on two calls in a row: the second call
finds the first call's leftovers in the shared array and must not be affected.
This file is collected last so that a run stopping at the first failure has run
every other test before it.
"""
import ctypes

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2e-3, 1e-4


def _case(seed, B, H, k, n, v, hot=0):
    idx, w = synth.random_selection(B, H, k, n * n, seed=seed, hot_rows=hot)
    g = synth.generator(seed + 1)
    values = (torch.randn(n * n, v, generator=g) / 16).to(torch.bfloat16)
    gout = torch.randn(B, v, generator=g).to(torch.bfloat16)
    return [t.cuda() for t in (values, idx, w, gout)]


def _regular(P, values, idx, w, gout, n):
    gv = torch.zeros(values.shape[0], values.shape[1], device="cuda")
    gs = torch.empty(idx.shape, device="cuda")
    P.pkm_backward_values(values, idx, w, gout, gv, gs, n)
    return gv, gs


def _noalloc(P, values, idx, w, gout, n):
    gv = torch.zeros(values.shape[0], values.shape[1], device="cuda")
    gs = torch.empty(idx.shape, device="cuda")
    B, H, k = idx.shape
    shape = P.make_shape(B, 0, H, 0, n, k, values.shape[1], values.dtype)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    rc = P.lib().pkm_backward_values_noalloc(ctypes.byref(shape), ptr(values), ptr(idx), ptr(w),
                                             ptr(gout), ptr(gv), ptr(gs), stream)
    assert rc == 0, P.pkm_status_string(rc)
    return gv, gs


def test_noalloc_matches_workspace_entry_point_twice():
    import product_key_memory_b200 as P
    cases = [_case(101, B=512, H=4, k=32, n=256, v=256),
             _case(202, B=300, H=2, k=16, n=128, v=512, hot=40)]
    for values, idx, w, gout in cases:        # two calls in a row, different inputs
        n = int(round(values.shape[0] ** 0.5))
        ref_gv, ref_gs = _regular(P, values, idx, w, gout, n)
        gv, gs = _noalloc(P, values, idx, w, gout, n)
        torch.cuda.synchronize()
        torch.testing.assert_close(gv, ref_gv, rtol=RTOL, atol=ATOL)
        torch.testing.assert_close(gs, ref_gs, rtol=RTOL, atol=ATOL)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import product_key_memory_b200 as P
    t = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    too_many_slots = P.make_shape(4, 0, 1, 0, 1025, 4, 8, 0)             # 1,050,625 slots
    too_many_picks = P.make_shape(70000, 0, 1, 0, 64, 32, 8, 0)          # 2,240,000 picks
    for s in (too_many_slots, too_many_picks):
        rc = P.lib().pkm_backward_values_noalloc(ctypes.byref(s), p, p, p, p, p, p, None)
        assert rc == -2                                                   # PKM_ERR_UNSUPPORTED
