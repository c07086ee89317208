"""pkm_slot_usage (distinct slots among a batch's picks) against the oracle's count."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _P():
    import product_key_memory_b200 as mod
    return mod


@pytest.mark.parametrize("B,H,k,n,hot", [(1, 1, 1, 4, 0), (300, 4, 32, 64, 0), (2000, 4, 32, 512, 0),
                                         (700, 2, 16, 128, 40), (64, 8, 32, 1024, 0)])
def test_slot_usage_matches_oracle(B, H, k, n, hot):
    idx, _ = synth.random_selection(B, H, k, n * n, seed=B + n, hot_rows=hot)
    got = int(_P().pkm_slot_usage(idx.cuda(), n).item())
    ref, bad = oracle.slot_usage(idx.numpy(), n * n)
    assert bad == 0 and got == ref


def test_slot_usage_of_forward_picks():
    w = synth.WORKLOADS["c512"].with_(B=512, n=256)
    L = synth.make_layer(w)
    d = {k: v.cuda() for k, v in L.items()}
    P = _P()
    _, idx, _, _ = P.pkm_forward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"],
                                 d["bn_beta"], d["subkeys"], d["values"], k=w.k)
    got = int(P.pkm_slot_usage(idx, w.n).item())
    assert got == oracle.slot_usage(idx.cpu().numpy(), w.n * w.n)[0]


def test_slot_usage_bad_ids_reported_and_skipped():
    P = _P()
    idx = torch.tensor([[[3, 3, 7, -1]], [[200, 7, 8, 9]]], dtype=torch.int32)  # n = 10: 100 slots
    shape = P.make_shape(2, 0, 1, 0, 10, 4, 8, 0)
    nb = int(P.lib().pkm_workspace_size(__import__("ctypes").byref(shape), 2))
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    hits = P.pkm_slot_usage(idx.cuda(), 10, workspace=ws)
    assert int(hits.item()) == 4                      # 3, 7, 8, 9
    assert P.pkm_device_status(ws) == -5


def test_slot_usage_no_tokens():
    P = _P()
    idx = torch.empty(0, 2, 4, dtype=torch.int32, device="cuda")
    assert int(P.pkm_slot_usage(idx, 16).item()) == 0
