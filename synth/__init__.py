"""Seeded synthetic inputs for the product-key memory (PKM) layer.

This module only draws random tensors of the right shapes, dtypes and
distributions. It holds none of the layer's arithmetic, so the fp64 oracle
(``oracle/``) and the CUDA library (``product_key_memory_b200``) can both take
their inputs from it without sharing any of the method.

Workloads (the shapes follow "Large Memory Layers with Product Keys": model dims
1024 and 1600, 512^2 and 1024^2 memory slots, H heads, k = 32):

=====  =====  =======  ==  ===  ====  ==  ====  =====
name   B      d_model  H   dq   n     k   v     dtype
=====  =====  =======  ==  ===  ====  ==  ====  =====
tiny   64     32       1   16   16    4   32    f32
c512   4096   1024     4   512  512   32  1024  bf16
c1024  16384  1024     4   512  1024  32  1024  bf16
wide   16384  1600     8   512  1024  32  1600  bf16
=====  =====  =======  ==  ===  ====  ==  ====  =====

``bwd512`` is the sparse value backward on ``c512`` with a bf16 ``grad_out``.

Distributions: "N(0, s)" means variance s. x ~ N(0, 1); W_q ~ N(0, 1/d_model);
BN running mean ~ N(0, 0.1) and running var ~ U(0.5, 2) (tiny: mean 0, var 1);
gamma = 1, beta = 0; sub-keys ~ N(0, 2/dq); values ~ N(0, 1/v). In ``wide`` the odd
rows of x are one of 64 seeded prototypes (N(0, 1)) plus N(0, 0.05) noise.
Every tensor is drawn in fp32 from one torch CPU generator (seed 20190710 + the
workload number) in a fixed order and rounded to bf16 (round to nearest even)
where the dtype is bf16.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

BASE_SEED = 20190710


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int
    B: int
    d_model: int
    H: int
    dq: int
    n: int
    k: int
    v: int
    dtype: str  # "f32" or "bf16"
    bn_random: bool = True
    prototypes: int = 0  # >0: odd rows of x come from this many prototypes

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def slots(self) -> int:
        return self.n * self.n

    def with_tokens(self, B: int) -> "Workload":
        return dataclasses.replace(self, B=B)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 0, B=64, d_model=32, H=1, dq=16, n=16, k=4, v=32,
                     dtype="f32", bn_random=False),
    "c512": Workload("c512", 1, B=4096, d_model=1024, H=4, dq=512, n=512, k=32,
                     v=1024, dtype="bf16"),
    "c1024": Workload("c1024", 2, B=16384, d_model=1024, H=4, dq=512, n=1024,
                      k=32, v=1024, dtype="bf16"),
    "wide": Workload("wide", 3, B=16384, d_model=1600, H=8, dq=512, n=1024,
                     k=32, v=1600, dtype="bf16", prototypes=64),
}
# The backward workload reuses the c512 layer.
BACKWARD_WORKLOAD = "bwd512"
BACKWARD_NUMBER = 4

_CHUNK = 1 << 24  # elements drawn per randn call for the large tables


def _normal(g: torch.Generator, shape, var: float, dtype) -> torch.Tensor:
    """N(0, var) drawn in fp32 chunks (bounded host memory), then cast."""
    numel = 1
    for s in shape:
        numel *= s
    out = torch.empty(numel, dtype=dtype)
    std = float(var) ** 0.5
    for lo in range(0, numel, _CHUNK):
        hi = min(numel, lo + _CHUNK)
        c = torch.randn(hi - lo, generator=g, dtype=torch.float32)
        c.mul_(std)
        out[lo:hi] = c.to(dtype)
    return out.view(*shape)


def generator(seed: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(int(seed))


def make_layer(w: Workload, seed: Optional[int] = None, with_values: bool = True):
    """Draw (x, W_q, BN stats, sub-keys, values) for workload ``w``.

    Returns a dict of CPU tensors:
      x        [B][d_model]        dtype
      W_q      [H*dq][d_model]     dtype   (q = x @ W_q^T)
      bn_mean, bn_var, bn_gamma, bn_beta  [H*dq] fp32
      subkeys  [H][2][n][dq/2]     dtype   ([h][0] = C, [h][1] = C')
      values   [n*n][v]            dtype
    """
    seed = BASE_SEED + w.number if seed is None else seed
    g = generator(seed)
    dt = w.torch_dtype
    F = w.H * w.dq
    x = _normal(g, (w.B, w.d_model), 1.0, torch.float32)
    if w.prototypes:
        protos = torch.randn(w.prototypes, w.d_model, generator=g)
        pick = torch.randint(0, w.prototypes, (w.B,), generator=g)
        noise = torch.randn(w.B, w.d_model, generator=g) * (0.05 ** 0.5)
        odd = torch.arange(w.B) % 2 == 1
        x[odd] = protos[pick[odd]] + noise[odd]
    x = x.to(dt)
    W_q = _normal(g, (F, w.d_model), 1.0 / w.d_model, dt)
    if w.bn_random:
        bn_mean = torch.randn(F, generator=g) * (0.1 ** 0.5)
        bn_var = torch.rand(F, generator=g) * 1.5 + 0.5
    else:
        bn_mean = torch.zeros(F)
        bn_var = torch.ones(F)
    bn_gamma = torch.ones(F)
    bn_beta = torch.zeros(F)
    subkeys = _normal(g, (w.H, 2, w.n, w.dq // 2), 2.0 / w.dq, dt)
    values = _normal(g, (w.slots, w.v), 1.0 / w.v, dt) if with_values else None
    return dict(x=x, W_q=W_q, bn_mean=bn_mean.float(), bn_var=bn_var.float(),
                bn_gamma=bn_gamma, bn_beta=bn_beta, subkeys=subkeys, values=values)


def make_grad_out(w: Workload, seed: Optional[int] = None) -> torch.Tensor:
    """grad_out [B][v] ~ N(0, 1) in the workload dtype (backward workload)."""
    seed = BASE_SEED + BACKWARD_NUMBER if seed is None else seed
    g = generator(seed + 7919)
    return _normal(g, (w.B, w.v), 1.0, w.torch_dtype)


def random_selection(B: int, H: int, k: int, slots: int, seed: int,
                     hot_rows: int = 0):
    """Seeded (indices, weights) for exercising the value backward on its own.

    indices [B][H][k] int32: k distinct slots per (token, head). With
    ``hot_rows`` >= k every pick comes from one pool of that many slots, so rows
    repeat across tokens heavily (the skewed case a sort-based scatter must handle).
    weights [B][H][k] fp32: positive, each (token, head) row sums to about 1.
    """
    g = generator(seed)
    if hot_rows:
        P = max(hot_rows, k)
        pool = torch.randperm(slots, generator=g)[:P]
        order = torch.rand(B, H, P, generator=g).argsort(-1)[..., :k]
        idx = pool[order]
    else:
        idx = torch.randint(0, slots, (B, H, k), generator=g)
        for _ in range(64):
            srt, _ = idx.sort(-1)
            dup = (srt[..., 1:] == srt[..., :-1]).any(-1)
            if not bool(dup.any()):
                break
            idx[dup] = torch.randint(0, slots, (int(dup.sum()), k), generator=g)
        else:  # pragma: no cover - needs slots close to k
            raise RuntimeError("could not draw distinct slots")
    w = torch.rand(B, H, k, generator=g) + 0.05
    w = w / w.sum(-1, keepdim=True)
    return idx.to(torch.int32), w.float()
