"""Host-side checks of the C ABI: the library loads, exports every entry point that
include/pkm.h declares, sizes workspaces, and rejects bad arguments before any
CUDA call (so these run without a GPU)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import product_key_memory_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "pkm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkm_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert "pkm_forward" in names and "pkm_backward_values" in names
    lib = ctypes.CDLL(P.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name
    assert set(P.EXPORTED) <= set(names)


def test_status_strings():
    for c in (0, -1, -2, -3, -4, -5):
        assert P.pkm_status_string(c)
    assert P.pkm_status_string(7) == "unknown status"


def _shape(**kw):
    base = dict(B=16384, d_model=1024, H=4, dq=512, n=1024, k=32, v=1024, dtype=1, bn_eps=1e-5)
    base.update(kw)
    return P.make_shape(**base)


def test_workspace_sizes():
    s = _shape()
    lists = 16384 * 4 * 2 * 32 * 8            # best 32 per half: fp32 score + int32 id
    fw = P.pkm_workspace_size(s)
    # tensor-core path: status + two bf16 q planes per token of a sub-batch + lists
    assert fw >= 256 + 16384 * 2048 * 4 + lists
    with P.options(subbatches=4):
        assert 256 + 4096 * 2048 * 4 + lists <= P.pkm_workspace_size(s) < fw
    with P.options(path="simt"):
        # CUDA-core path: fp32 q for every token
        assert P.pkm_workspace_size(s) >= 256 + 16384 * 2048 * 4 + lists
    assert P.pkm_workspace_size(s) == fw
    bw = P.pkm_workspace_size(s, True)
    assert bw >= 256 + 4 * (2 * 1024 * 1024 + 16384 * 4 * 32)
    assert P.pkm_workspace_size(_shape(B=0)) > 0


def _a256(x):
    return (x + 255) // 256 * 256


def _small_ws(B, H, dq, n, v):
    """Forward workspace of the small-batch path: status, fp32 q, chunk lists (one list
    of 32 per 64-sub-key chunk of each half), per-head rows and per-token counts."""
    L = B * H * 2 * ((n + 63) // 64) * 32
    return 256 + _a256(B * H * dq * 4) + 2 * _a256(L * 4) + _a256(B * H * v * 4 + B * 4)


@pytest.mark.parametrize("name,cut", [("c1024", 384), ("c512", 384), ("wide", 240),
                                      ("tiny", 112)])
def test_automatic_small_batch_cut_off(name, cut):
    """The default choice sends batches up to the cut-off to the small-batch kernels (384
    tokens with H <= 4 and 240 with H = 8 on bf16 layers with tensor-core tiles, 112
    with H <= 4 otherwise) and larger ones elsewhere; a pinned small-batch form takes up
    to 512 tokens. The forward's workspace layout tells the paths apart."""
    import synth
    w = synth.WORKLOADS[name]
    dt = 1 if w.dtype == "bf16" else 0

    def ws(B):
        return P.pkm_workspace_size(_shape(B=B, d_model=w.d_model, H=w.H, dq=w.dq, n=w.n,
                                           k=w.k, v=w.v, dtype=dt))

    for B in (1, 9, cut):
        assert ws(B) == _small_ws(B, w.H, w.dq, w.n, w.v), B
    assert ws(cut + 1) != _small_ws(cut + 1, w.H, w.dq, w.n, w.v)
    with P.options(path="small_split"):
        assert ws(512) == _small_ws(512, w.H, w.dq, w.n, w.v)
        assert ws(513) != _small_ws(513, w.H, w.dq, w.n, w.v)


def test_options_set_get_and_reject():
    assert P.pkm_get_option(P.PKM_OPT_PATH) == P.PKM_PATH_AUTO
    assert P.pkm_get_option(P.PKM_OPT_SUBBATCHES) == 1
    with P.options(path="tc", subbatches=3):
        assert P.pkm_get_option(P.PKM_OPT_PATH) == P.PKM_PATH_TC
        assert P.pkm_get_option(P.PKM_OPT_SUBBATCHES) == 3
    assert P.pkm_get_option(P.PKM_OPT_PATH) == P.PKM_PATH_AUTO
    assert P.pkm_get_option(P.PKM_OPT_SUBBATCHES) == 1
    L = P.lib()
    assert L.pkm_set_option(P.PKM_OPT_PATH, 7) == -1
    assert L.pkm_set_option(P.PKM_OPT_SUBBATCHES, 0) == -1
    assert L.pkm_set_option(P.PKM_OPT_SUBBATCHES, 5) == -1
    assert L.pkm_set_option(9, 1) == -1
    assert L.pkm_get_option(9) == -1
    assert P.pkm_get_option(P.PKM_OPT_SUBBATCHES) == 1


def test_environment_gives_initial_options():
    """PKM_PATH / PKM_SUBBATCHES are read once, as the initial option values."""
    code = ("import product_key_memory_b200 as P; "
            "print(P.pkm_get_option(P.PKM_OPT_PATH), P.pkm_get_option(P.PKM_OPT_SUBBATCHES))")
    env = dict(os.environ, PKM_PATH="simt", PKM_SUBBATCHES="3", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["2", "3"]


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), -1), (dict(k=33, n=64), -2), (dict(k=8, n=4), -1), (dict(dq=7), -1),
    (dict(H=0), -1), (dict(v=0), -1), (dict(dtype=3), -1), (dict(n=46341), -1),
    (dict(v=1001), -2), (dict(bn_eps=-1.0), -1), (dict(B=-1), -1),
])
def test_invalid_shapes_rejected_without_launch(kw, code):
    s = _shape(**kw)
    assert P.pkm_workspace_size(s) == 0
    fake = ctypes.c_void_p(1 << 20)
    rc = P.lib().pkm_forward(ctypes.byref(s), *([fake] * 12), fake, 1 << 40, None)
    assert rc == code


def test_null_and_misaligned_pointers_rejected():
    s = _shape(B=4)
    ok = ctypes.c_void_p(1 << 20)
    args = [ok] * 12
    args[3] = None                                 # bn_var
    assert P.lib().pkm_forward(ctypes.byref(s), *args, ok, 1 << 40, None) == -1
    args = [ok] * 12
    args[7] = ctypes.c_void_p((1 << 20) + 8)       # values not 16-byte aligned
    assert P.lib().pkm_forward(ctypes.byref(s), *args, ok, 1 << 40, None) == -2
    args = [ok] * 12
    assert P.lib().pkm_forward(ctypes.byref(s), *args, ok, 100, None) == -3          # small
    assert P.lib().pkm_forward(ctypes.byref(s), *args, ctypes.c_void_p((1 << 20) + 16),
                               1 << 40, None) == -3                                     # unaligned
    assert P.lib().pkm_backward_values(ctypes.byref(s), *([ok] * 6), ok, 10, None) == -3


def test_null_shape_rejected():
    assert P.lib().pkm_workspace_size(None, 0) == 0
    ok = ctypes.c_void_p(1 << 20)
    assert P.lib().pkm_forward(None, *([ok] * 13), 1 << 40, None) == -1


def test_zero_tokens_accepts_null_per_token_pointers():
    s = _shape(B=0)
    ok = ctypes.c_void_p(1 << 20)
    args = [None, ok, ok, ok, ok, ok, ok, ok, None, None, None, None]   # x, out, idx, w, scores NULL
    assert P.lib().pkm_forward(ctypes.byref(s), *args, ok, 1 << 40, None) == 0
    bargs = [ok, None, None, None, ok, None]     # values, indices, weights, grad_out, grad_values, grad_scores
    assert P.lib().pkm_backward_values(ctypes.byref(s), *bargs, ok, 1 << 40, None) == 0
    s4 = _shape(B=4)
    assert P.lib().pkm_forward(ctypes.byref(s4), *args, ok, 1 << 40, None) == -1


def test_full_backward_workspace_and_argument_checks():
    s = _shape(B=4096, n=512)
    need = P.lib().pkm_workspace_size(ctypes.byref(s), 3)
    E = 4096 * 4 * 32
    # kept-score grads + acc, dL/dq, dL/dacc + q planes + sub-key targets and order
    assert need >= 256 + 4 * E + 3 * 4 * 4096 * 2048 + 6 * 4096 * 2048 + 2 * 4 * 2 * E
    assert P.lib().pkm_workspace_size(ctypes.byref(_shape(dq=7)), 3) == 0
    ok = ctypes.c_void_p(1 << 20)
    args = [ok] * 11 + [None] * 7                   # inputs, no gradients requested
    bad = list(args)
    bad[1] = None                                   # W_q
    assert P.lib().pkm_backward(ctypes.byref(s), *bad, ok, 1 << 40, None) == -1
    bad = list(args)
    bad[6] = ctypes.c_void_p((1 << 20) + 4)         # sub-keys misaligned
    assert P.lib().pkm_backward(ctypes.byref(s), *bad, ok, 1 << 40, None) == -2
    assert P.lib().pkm_backward(ctypes.byref(s), *args, ok, 100, None) == -3
    s0 = _shape(B=0)
    zargs = [None, ok, ok, ok, ok, ok, ok, ok, None, None, None] + [None] * 7
    assert P.lib().pkm_backward(ctypes.byref(s0), *zargs, ok, 1 << 40, None) == 0


def test_training_bn_entry_points_validate_before_launch():
    s = _shape(B=4096, n=512)
    fw = P.lib().pkm_workspace_size(ctypes.byref(s), 4)
    # forward workspace + acc of the whole batch (three bf16 planes) + fp64 chunk stats
    assert fw >= P.pkm_workspace_size(s) + 4096 * 2048 * 6 + 32 * 2 * 2048 * 8
    assert P.lib().pkm_workspace_size(ctypes.byref(_shape(B=1)), 4) == 0
    ok = ctypes.c_void_p(1 << 20)
    f = P.lib().pkm_forward_train
    args = [ok] * 6 + [ctypes.c_float(0.1)] + [ok] * 8   # through batch_var
    assert f(ctypes.byref(_shape(B=1)), *args, ok, 1 << 40, None) == -1        # one token
    bad = list(args)
    bad[6] = ctypes.c_float(1.5)                                                 # momentum
    assert f(ctypes.byref(s), *bad, ok, 1 << 40, None) == -1
    bad = list(args)
    bad[14] = None                                                               # batch_var
    assert f(ctypes.byref(s), *bad, ok, 1 << 40, None) == -1
    assert f(ctypes.byref(s), *args, ok, 100, None) == -3
    bargs = [ok] * 11 + [None] * 7
    assert P.lib().pkm_backward_train(ctypes.byref(_shape(B=1)), *bargs, ok, 1 << 40, None) == -1
    assert P.lib().pkm_backward_train(ctypes.byref(s), *bargs, ok, 100, None) == -3


def test_no_cpu_fallback_host_tensors_are_refused():
    """The binding hands only device pointers to the library: CPU tensors raise
    instead of running anywhere else."""
    import torch
    x = torch.zeros(4, 32)
    with pytest.raises(ValueError, match="device tensors"):
        P.pkm_forward(x, torch.zeros(16, 32), torch.zeros(16), torch.ones(16), torch.ones(16),
                      torch.zeros(16), torch.zeros(1, 2, 16, 8), torch.zeros(256, 32), k=4)


def test_missing_library_fails_loudly():
    import subprocess
    import sys
    # The package loads the library when it is imported.
    code = ("try:\n    import product_key_memory_b200\n"
            "except ImportError as e:\n    print('raised', e)\n")
    env = dict(os.environ, PKM_LIBRARY=os.path.join(ROOT, "no_such_library.so"))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=120)
    assert "raised" in r.stdout and "not built" in r.stdout, r.stdout + r.stderr


def test_full_backward_rejects_more_picks_than_32_bit_positions():
    # 2 * B * H * k contributions must fit the sort's 32-bit positions.
    s = _shape(B=(1 << 30) // (4 * 32) + 1, n=512)
    assert P.lib().pkm_workspace_size(ctypes.byref(s), 3) == 0
    ok = ctypes.c_void_p(1 << 20)
    assert P.lib().pkm_backward(ctypes.byref(s), *([ok] * 11), *([None] * 7), ok, 1 << 40,
                                None) == -2
