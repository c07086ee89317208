"""The timeout path of the tensor-core kernels, run on the GPU without a hang.

The test build of the library (libpkm_waittest.so: every pipeline wait gives up as
soon as one try does not satisfy it, so the first wait on a copy from HBM always runs
out; the drains keep their full second) is loaded in a child process through
PKM_LIBRARY. Its forward and full backward must return, record the timeout in the
workspace status word (pkm_device_status -> PKM_ERR_DEVICE), leave the CUDA context
usable, and exit cleanly. Nothing is done to the GPU that a normal call does not do:
the waits end early and the kernels drain their own copies and MMAs before exiting.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WAITTEST = os.path.join(ROOT, "product_key_memory_b200", "libpkm_waittest.so")

CHILD = r"""
import sys, torch
sys.path.insert(0, ROOT)
import synth
import product_key_memory_b200 as P
assert P.LIB_PATH.endswith("libpkm_waittest.so"), P.LIB_PATH
w = synth.WORKLOADS["c512"].with_(B=1024)
L = {k: v.cuda() for k, v in synth.make_layer(w).items()}
shape = P.make_shape(w.B, w.d_model, w.H, w.dq, w.n, w.k, w.v, torch.bfloat16)
ws = torch.zeros(P.pkm_workspace_size(shape), dtype=torch.uint8, device="cuda")
out, idx, wt, _ = P.pkm_forward(L["x"], L["W_q"], L["bn_mean"], L["bn_var"], L["bn_gamma"],
                                L["bn_beta"], L["subkeys"], L["values"], k=w.k, workspace=ws)
fwd = P.pkm_device_status(ws)
grads = {"x": torch.empty(w.B, w.d_model, device="cuda"),
         "W_q": torch.empty(w.H * w.dq, w.d_model, device="cuda")}
idx.clamp_(0, w.n * w.n - 1)
nb = int(P.lib().pkm_workspace_size(__import__("ctypes").byref(shape), 3))
bws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
P.pkm_backward(L["x"], L["W_q"], L["bn_mean"], L["bn_var"], L["bn_gamma"], L["bn_beta"],
               L["subkeys"], L["values"], idx, wt.nan_to_num(0.0), synth.make_grad_out(w).cuda(),
               grads, workspace=bws)
bwd = P.pkm_device_status(bws)
torch.cuda.synchronize()
# The context is still usable: an ordinary torch kernel and copy.
assert float((torch.ones(1000, device="cuda") * 2).sum().item()) == 2000.0
print("STATUS", fwd, bwd, flush=True)
""".replace("ROOT", repr(ROOT))


@pytest.mark.skipif(not os.path.exists(WAITTEST), reason="test build not built")
def test_pipeline_waits_time_out_and_report():
    env = dict(os.environ, PKM_LIBRARY=WAITTEST)
    env.pop("PKM_PATH", None)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("STATUS")][-1]
    fwd, bwd = (int(v) for v in line.split()[1:])
    assert fwd == -5 and bwd == -5, line       # PKM_ERR_DEVICE: the timeout was recorded


def test_normal_build_still_clean_after():
    """The regular library in this process: a forward reports no device error."""
    import torch
    import synth
    import product_key_memory_b200 as P
    w = synth.WORKLOADS["c512"].with_(B=256, n=256)
    L = {k: v.cuda() for k, v in synth.make_layer(w).items()}
    shape = P.make_shape(w.B, w.d_model, w.H, w.dq, w.n, w.k, w.v, torch.bfloat16)
    ws = torch.zeros(P.pkm_workspace_size(shape), dtype=torch.uint8, device="cuda")
    P.pkm_forward(L["x"], L["W_q"], L["bn_mean"], L["bn_var"], L["bn_gamma"], L["bn_beta"],
                  L["subkeys"], L["values"], k=w.k, workspace=ws)
    assert P.pkm_device_status(ws) == 0
