"""Seeded synthetic inputs for the SSD layer.

This module is the one piece that both the CUDA path's callers (tests,
benchmark) and the fp64 oracle's tests use.  It draws random numbers and
rounds them to the storage dtype; it holds none of the layer's arithmetic.

Value recipe (the same for every workload):
    x ~ N(0, 1)                     stored in the workload dtype (bf16 or fp32)
    dt = softplus(z), z ~ N(-4, 0.5)    fp32, already positive (the layer applies no softplus)
    A_h = -exp(u), u ~ U(ln 1, ln 16)   fp32, one scalar per head, in [-16, -1]
    B, C ~ N(0, 1) / sqrt(N)        stored in the workload dtype (scale applied before rounding)
    D_h ~ N(0, 1)                   fp32
    init ~ N(0, 0.1^2)              fp32 (standard deviation 0.1), only where a workload asks for it

Draw order from one ``torch.Generator``: x, z, A, B, C, D, init.  Workload
shapes follow the 130M / 2.7B Mamba-2 layer shapes and the N=64 length sweep
(the speed comparison on the "Transformers are SSMs" CiteArk page, claim on
A100-80GB PCIe, L = 512 ... 512K).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str          # "f32" or "bf16": storage type of x, B, C and y
    with_init: bool     # random initial states are passed
    want_final: bool    # final states are requested
    seed: int

    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _sweep(L: int) -> Workload:
    return Workload(f"sweep_n64_L{L}", batch=(512 * 1024) // L, seqlen=L, nheads=32, headdim=64,
                    dstate=64, ngroups=1, chunk=256, dtype="bf16", with_init=False,
                    want_final=False, seed=1234 + 3000 + int(math.log2(L)))


# Named workloads (seeds 1234 + index; the sweep uses 1234 + 3000 + log2 L).
TINY_F32 = Workload("tiny_f32_b1_L256_H4_P16_N16", 1, 256, 4, 16, 16, 1, 64, "f32",
                    with_init=False, want_final=True, seed=1234)
LAYER_130M = Workload("mamba2_130m_layer_b8_L2048_H24_P64_N128", 8, 2048, 24, 64, 128, 1, 256,
                      "bf16", with_init=False, want_final=False, seed=1235)
LAYER_2P7B = Workload("mamba2_2p7b_layer_b4_L8192_H80_P64_N128", 4, 8192, 80, 64, 128, 1, 256,
                      "bf16", with_init=True, want_final=True, seed=1236)
SWEEP_LENGTHS = (512, 2048, 8192, 32768, 131072, 524288)
SWEEP = tuple(_sweep(L) for L in SWEEP_LENGTHS)


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    steps: int
    dtype: str
    seed: int


DECODE_2P7B = DecodeWorkload("decode_b256_H80_P64_N128", 256, 80, 64, 128, 1, 1024, "bf16",
                             seed=1238)


def _normal(shape, gen, device, std=1.0, mean=0.0):
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def make_inputs(w: Workload, device="cpu", gen: torch.Generator | None = None):
    """Draw one workload's inputs.  Returns a dict of tensors on ``device``:
    x, dt, A, B, C, D and init (None unless ``w.with_init``).  x, B, C are in
    the workload dtype; everything else is fp32."""
    if gen is None:
        gen = torch.Generator(device=device)
        gen.manual_seed(w.seed)
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    st = w.torch_dtype()
    x = _normal((b, L, H, P), gen, device).to(st)
    z = _normal((b, L, H), gen, device, std=0.5, mean=-4.0)
    dt = torch.nn.functional.softplus(z)
    u = torch.rand(H, generator=gen, device=device, dtype=torch.float32) * math.log(16.0)
    A = -torch.exp(u)
    Bm = _normal((b, L, G, N), gen, device, std=1.0 / math.sqrt(N)).to(st)
    Cm = _normal((b, L, G, N), gen, device, std=1.0 / math.sqrt(N)).to(st)
    D = _normal((H,), gen, device)
    init = _normal((b, H, P, N), gen, device, std=0.1) if w.with_init else None
    return {"x": x, "dt": dt, "A": A, "B": Bm, "C": Cm, "D": D, "init": init}


def make_decode_params(w: DecodeWorkload, device="cpu", gen: torch.Generator | None = None):
    """Per-layer decode parameters and the starting state: returns
    (gen, dict(A, D, state)).  The same generator then feeds
    ``make_decode_token`` once per step, in step order."""
    if gen is None:
        gen = torch.Generator(device=device)
        gen.manual_seed(w.seed)
    H, P, N = w.nheads, w.headdim, w.dstate
    u = torch.rand(H, generator=gen, device=device, dtype=torch.float32) * math.log(16.0)
    A = -torch.exp(u)
    D = _normal((H,), gen, device)
    state = _normal((w.batch, H, P, N), gen, device, std=0.1)
    return gen, {"A": A, "D": D, "state": state}


def make_decode_token(w: DecodeWorkload, gen: torch.Generator, device="cpu"):
    """One decode step's per-token inputs (x, dt, B, C), drawn in that order."""
    st = torch.float32 if w.dtype == "f32" else torch.bfloat16
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    x = _normal((b, H, P), gen, device).to(st)
    z = _normal((b, H), gen, device, std=0.5, mean=-4.0)
    dt = torch.nn.functional.softplus(z)
    Bm = _normal((b, G, N), gen, device, std=1.0 / math.sqrt(N)).to(st)
    Cm = _normal((b, G, N), gen, device, std=1.0 / math.sqrt(N)).to(st)
    return {"x": x, "dt": dt, "B": Bm, "C": Cm}
