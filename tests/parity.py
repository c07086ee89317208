"""Comparison of the CUDA library's outputs with the fp64 oracle.

Rules (stated with each test's tolerance):
* indices: equal position by position, except where the GPU's pick and the
  oracle's pick at that position have fp64 scores within REL_TIE * max(|S_k|, 1e-6)
  of each other (S_k = the oracle's k-th kept score). Such (token, head) pairs are
  "exempt": near-ties that fp32 arithmetic may order either way. They are counted.
  Picks must always be distinct and inside [0, n*n).
* weights / scores / out: |gpu - ref| <= ATOL + RTOL * |ref| elementwise. For a
  token with an exempt head the reference is the oracle's softmax and value sum
  re-run on the GPU's picks (with the oracle's fp64 scores of those picks).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

RTOL = 2e-3
ATOL = 1e-4
REL_TIE = 1e-5


def allclose_report(name, got, ref, rtol=RTOL, atol=ATOL):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        i = np.unravel_index(np.argmax(err - (atol + rtol * np.abs(ref))), err.shape)
        raise AssertionError("%s: %d of %d elements out of tolerance; worst at %s: got %r ref %r"
                             % (name, int(bad.sum()), bad.size, i, got[i], ref[i]))
    return float(err.max()) if err.size else 0.0


def grad_report(name, got, ref, rtol=RTOL, atol=ATOL):
    """Gradient tensor against the oracle with the stated bar |got - ref| <=
    atol + rtol |ref| elementwise (no scaling with the tensor's size). Prints and
    returns the worst error as a fraction of its element's bar (<= 1 passes)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64).reshape(got.shape)
    allclose_report(name, got, ref, rtol, atol)
    frac = float((np.abs(got - ref) / (atol + rtol * np.abs(ref))).max()) if got.size else 0.0
    print("%s: worst error %.3g of the bar, max |ref| %.3g" % (
        name, frac, float(np.abs(ref).max()) if ref.size else 0.0))
    return frac


def compare_forward(gpu: dict, ref: dict, values_cpu: torch.Tensor, n: int, *,
                    rtol=RTOL, atol=ATOL, rel_tie=REL_TIE, max_exempt_frac=0.01):
    """gpu: numpy out/indices/weights/scores for the same tokens as ref (oracle with
    want_half=True). Returns a dict of statistics (exempt count, max errors)."""
    gi = gpu["indices"].astype(np.int64)
    ri = ref["indices"].astype(np.int64)
    B, H, k = ri.shape
    half = ref["half"]                                      # [B][H][2][n]
    assert ((gi >= 0) & (gi < n * n)).all(), "GPU pick outside [0, n*n)"
    srt = np.sort(gi, axis=-1)
    assert not (srt[..., 1:] == srt[..., :-1]).any(), "GPU picks repeat within a (token, head)"
    tt = np.arange(B)[:, None, None]
    hh = np.arange(H)[None, :, None]
    sg = half[tt, hh, 0, gi // n] + half[tt, hh, 1, gi % n]   # fp64 score of each GPU pick
    s_k = np.abs(ref["scores"][..., -1:])
    tol = rel_tie * np.maximum(s_k, 1e-6)
    same = gi == ri
    near = np.abs(sg - ref["scores"]) <= tol
    ok = same | near
    if not ok.all():
        t, h, j = np.argwhere(~ok)[0]
        raise AssertionError(
            "index mismatch at token %d head %d pos %d: gpu %d (score %r) vs oracle %d (score %r); "
            "%d positions differ beyond the tie window" % (t, h, j, gi[t, h, j], sg[t, h, j],
                                                         ri[t, h, j], ref["scores"][t, h, j],
                                                         int((~ok).sum())))
    exempt_th = ~same.all(-1)                                 # [B][H]
    n_exempt = int(exempt_th.sum())
    assert n_exempt <= max(2, max_exempt_frac * B * H), "too many exempt (token, head): %d" % n_exempt
    ref_w = ref["weights"].copy()
    ref_s = ref["scores"].copy()
    ref_out = ref["out"].copy() if ref.get("out") is not None else None
    tok = np.nonzero(exempt_th.any(-1))[0]
    if tok.size:
        w2, o2 = oracle.finish(sg[tok], gi[tok].astype(np.int32), values_cpu)
        ref_w[tok] = w2
        ref_s[tok] = sg[tok]
        if ref_out is not None:
            ref_out[tok] = o2
    stats = dict(exempt=n_exempt, pairs=B * H)
    stats["err_w"] = allclose_report("weights", gpu["weights"], ref_w, rtol, atol)
    if gpu.get("scores") is not None:
        stats["err_s"] = allclose_report("scores", gpu["scores"], ref_s, rtol, atol)
    if ref_out is not None:
        stats["err_out"] = allclose_report("out", gpu["out"], ref_out, rtol, atol)
    return stats


def to_numpy(out, idx, w, s):
    return dict(out=out.float().cpu().numpy(), indices=idx.cpu().numpy(),
                weights=w.cpu().numpy(), scores=None if s is None else s.cpu().numpy())
