"""Seeded synthetic inputs for the selective scan, shared by the CUDA path's
tests/bench and by the fp64 oracle.

This module holds none of the method's arithmetic: it only draws random
numbers, rounds them to the storage type (bf16 round-to-nearest-even, done
here on the host so that both sides see the very same values) and widens
bf16 back to fp32 (exact).  The step-size bias is chosen with the inverse of
softplus so that the step sizes land in the stated range; that inverse is
input construction only, never part of either computation.

Recipe (the same for every workload; the seed is fixed per workload):

* u, z, B, C ~ N(0, 1)
* delta_raw = 0.1 * N(0, 1)
* bias[d] = softplus^-1(dt_d) = log(expm1(dt_d)),  dt_d = exp(U(ln 1e-3, ln 1e-1)),
  so that softplus(delta_raw + bias) is log-uniform on about [1e-3, 1e-1]
* A[d, n] = -(n + 1)  (the S4D-Real initialisation with negative real poles);
  other A recipes (tests only): "scaled" A[d, n] = -(n + 1) * s_d with
  s_d = exp(U(ln 0.5, ln 2)) per channel (the product rounded in fp32, so the
  rows stay exactly geometric); "random" A[d, n] = -exp(U(ln 0.1, ln 20)) per
  channel and state; "mixed" cycles channel by channel through the S4D-Real,
  random and scaled rows, so that every group of consecutive channels holds
  all three kinds
* D = 1, or D ~ N(1, 0.1) where the workload says so
* everything is drawn in fp32, then rounded to bf16 for bf16 workloads;
  A, D and bias stay fp32.

With the causal convolution in front of the scan, u is read as the
convolution's input x (the same N(0, 1) draws), the taps are
conv_w ~ N(0, 0.5^2) and conv_b ~ N(0, 0.1^2) (fp32), and a conv state (the
inputs before the first token) is N(0, 1) in the io type.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int
    dstate: int
    seqlen: int          # 0 for a decode workload
    dtype: str           # "f32" or "bf16"
    d_skip: str          # "one" or "normal"
    seed: int
    decode_steps: int = 0

    @property
    def channel_tokens(self) -> int:
        return self.batch * self.dim * max(self.seqlen, 1)


# Named by what they are, with their sizes.  Seeds are 1000 + the workload's
# position in the list.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("s6-fwd-fp32-b1-d16-n4-l256", 1, 16, 4, 256, "f32", "one", 1001),
        Workload("mamba130m-layer-bf16-b8-d1536-n16-l2048", 8, 1536, 16, 2048, "bf16", "one", 1002),
        Workload("mamba1.4b-layer-bf16-b4-d4096-n16-l4096", 4, 4096, 16, 4096, "bf16", "normal", 1003),
        Workload("long-seq-bf16-b1-d2048-n16-l131072", 1, 2048, 16, 131072, "bf16", "one", 1004),
        Workload("decode-bf16-b256-d5120-n16-x1024", 256, 5120, 16, 0, "bf16", "normal", 1005,
                 decode_steps=1024),
    ]
}

FWD_WORKLOADS = [n for n, w in WORKLOADS.items() if w.seqlen > 0]
BENCH_WORKLOAD = "mamba1.4b-layer-bf16-b4-d4096-n16-l4096"
DECODE_WORKLOAD = "decode-bf16-b256-d5120-n16-x1024"


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns the
    16-bit patterns as uint16.  Inputs here are finite."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Tensor:
    """One input tensor: the values both sides compute on (fp32, exact) and the
    bytes the device receives (fp32 values, or bf16 bit patterns)."""
    values: np.ndarray       # float32
    stored: np.ndarray       # float32 or uint16 (bf16 bits)
    dtype: str               # "f32" or "bf16"


def _store(x32: np.ndarray, dtype: str) -> Tensor:
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "f32":
        return Tensor(x32, x32, "f32")
    if dtype == "bf16":
        bits = to_bf16_bits(x32)
        return Tensor(bf16_bits_to_f32(bits), bits, "bf16")
    raise ValueError(f"unknown dtype {dtype!r}")


def _rng(seed, *stream):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, stream)])))


A_RECIPES = ("s4d-real", "scaled", "random", "mixed")


def a_matrix(dim: int, dstate: int, recipe: str, seed: int) -> np.ndarray:
    """A [dim, N] fp32 (negative values) by recipe; see the module docstring."""
    s4d = -np.broadcast_to(np.arange(1, dstate + 1, dtype=np.float32), (dim, dstate)).copy()
    if recipe == "s4d-real":
        return s4d
    if recipe not in A_RECIPES:
        raise ValueError(f"unknown A recipe {recipe!r}")
    rng = _rng(seed, 8)
    scale = np.exp(rng.uniform(np.log(0.5), np.log(2.0), size=(dim, 1))).astype(np.float32)
    scaled = (s4d * scale).astype(np.float32)          # fp32 products: exactly (n+1) * A[d, 0]
    rand = (-np.exp(rng.uniform(np.log(0.1), np.log(20.0), size=(dim, dstate)))).astype(np.float32)
    if recipe == "scaled":
        return scaled
    if recipe == "random":
        return rand
    kind = np.arange(dim) % 3
    return np.where((kind == 0)[:, None], s4d, np.where((kind == 1)[:, None], rand, scaled)).astype(np.float32)


def channel_params(dim: int, dstate: int, d_skip: str, seed: int, a_init: str = "s4d-real"):
    """A [dim, N], D [dim], bias [dim] -- fp32."""
    rng = _rng(seed, 0)
    A = a_matrix(dim, dstate, a_init, seed)
    log_dt = rng.uniform(np.log(1e-3), np.log(1e-1), size=dim)
    dt = np.exp(log_dt)
    bias = np.log(np.expm1(dt)).astype(np.float32)
    if d_skip == "one":
        D = np.ones(dim, dtype=np.float32)
    elif d_skip == "normal":
        D = (1.0 + 0.1 * rng.standard_normal(dim)).astype(np.float32)
    else:
        raise ValueError(f"unknown D recipe {d_skip!r}")
    return A, D, bias


def scan_inputs(batch: int, dim: int, dstate: int, seqlen: int, dtype: str,
                seed: int, d_skip: str = "one", a_init: str = "s4d-real") -> dict:
    """Inputs of one forward pass.  u, delta, z: [batch, dim, L]; B, C:
    [batch, N, L]; A: [dim, N]; D, delta_bias: [dim]."""
    A, D, bias = channel_params(dim, dstate, d_skip, seed, a_init)
    rng = _rng(seed, 1)
    shape = (batch, dim, seqlen)
    u = _store(rng.standard_normal(shape, dtype=np.float32), dtype)
    delta = _store(np.float32(0.1) * rng.standard_normal(shape, dtype=np.float32), dtype)
    z = _store(rng.standard_normal(shape, dtype=np.float32), dtype)
    B = _store(rng.standard_normal((batch, dstate, seqlen), dtype=np.float32), dtype)
    C = _store(rng.standard_normal((batch, dstate, seqlen), dtype=np.float32), dtype)
    return dict(u=u, delta=delta, z=z, B=B, C=C, A=A, D=D, delta_bias=bias,
                batch=batch, dim=dim, dstate=dstate, seqlen=seqlen, dtype=dtype)


def workload_inputs(name: str, seqlen: Optional[int] = None) -> dict:
    w = WORKLOADS[name]
    if w.seqlen == 0:
        raise ValueError(f"{name} is a decode workload; use decode_step_inputs")
    return scan_inputs(w.batch, w.dim, w.dstate, w.seqlen if seqlen is None else seqlen,
                       w.dtype, w.seed, w.d_skip)


def decode_step_inputs(batch: int, dim: int, dstate: int, dtype: str, seed: int,
                       step: int) -> dict:
    """Per-token inputs of decode step `step`: u, delta, z [batch, dim];
    B, C [batch, N].  Each step draws from its own seeded stream."""
    rng = _rng(seed, 2, step)
    u = _store(rng.standard_normal((batch, dim), dtype=np.float32), dtype)
    delta = _store(np.float32(0.1) * rng.standard_normal((batch, dim), dtype=np.float32), dtype)
    z = _store(rng.standard_normal((batch, dim), dtype=np.float32), dtype)
    B = _store(rng.standard_normal((batch, dstate), dtype=np.float32), dtype)
    C = _store(rng.standard_normal((batch, dstate), dtype=np.float32), dtype)
    return dict(u=u, delta=delta, z=z, B=B, C=C)


def initial_state(batch: int, dim: int, dstate: int, seed: int, kind: str = "zero") -> np.ndarray:
    """fp32 starting state [batch, dim, N]: zeros, or N(0, 1) draws."""
    if kind == "zero":
        return np.zeros((batch, dim, dstate), dtype=np.float32)
    if kind == "normal":
        return _rng(seed, 3).standard_normal((batch, dim, dstate), dtype=np.float32)
    raise ValueError(f"unknown initial state {kind!r}")


def conv_params(dim: int, width: int, seed: int):
    """Causal convolution taps [dim, width] and bias [dim], fp32."""
    rng = _rng(seed, 4)
    w = (np.float32(0.5) * rng.standard_normal((dim, width), dtype=np.float32)).astype(np.float32)
    b = (np.float32(0.1) * rng.standard_normal(dim, dtype=np.float32)).astype(np.float32)
    return w, b


def conv_state(batch: int, dim: int, width: int, dtype: str, seed: int) -> Tensor:
    """The width-1 inputs before the first token, [batch, dim, width-1]."""
    return _store(_rng(seed, 5).standard_normal((batch, dim, width - 1), dtype=np.float32), dtype)


def upstream_gradients(batch: int, dim: int, dstate: int, seqlen: int, dtype: str, seed: int):
    """Gradients arriving at the backward pass: dy ~ N(0, 1) [batch, dim, L]
    in the io type, dlast ~ N(0, 1) [batch, dim, N] fp32."""
    rng = _rng(seed, 6)
    dy = _store(rng.standard_normal((batch, dim, seqlen), dtype=np.float32), dtype)
    dlast = rng.standard_normal((batch, dim, dstate), dtype=np.float32)
    return dy, dlast


# The structured-state-space-duality (Mamba-2) layer: token-major tensors,
# a scalar A per head, heads sharing B and C within a group.
SSD_WORKLOAD = "mamba2-layer-bf16-b4-l4096-h64-p64-n128-g1"
# a second layer shape: 80 heads of 64 (d_inner 5120), two sequences
SSD_WORKLOAD_2 = "mamba2-layer-bf16-b2-l4096-h80-p64-n128-g1"
SSD_SHAPES = {SSD_WORKLOAD: dict(batch=4, seqlen=4096, nheads=64, headdim=64, ngroups=1, dstate=128, seed=1006),
              SSD_WORKLOAD_2: dict(batch=2, seqlen=4096, nheads=80, headdim=64, ngroups=1, dstate=128, seed=1007)}


def ssd_inputs(batch: int, seqlen: int, nheads: int, headdim: int, ngroups: int, dstate: int, seed: int,
               dtype: str = "bf16") -> dict:
    """x, z ~ N(0, 1) [batch, L, H, P]; dt_raw = 0.1 N(0, 1) [batch, L, H] with
    dt_bias = softplus^-1 of a log-uniform step on [1e-3, 1e-1] per head;
    A_h = -exp(U(0, ln 16)); B, C ~ N(0, 1) / sqrt(N) [batch, L, G, N] (so that
    C . B stays of order one); D ~ N(1, 0.1).  bf16 storage for x, z, dt, B, C."""
    rng = _rng(seed, 7)
    f = lambda *s: rng.standard_normal(s, dtype=np.float32)
    dt_h = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), size=nheads))
    scale = np.float32(1.0 / np.sqrt(dstate))
    return dict(
        x=_store(f(batch, seqlen, nheads, headdim), dtype),
        z=_store(f(batch, seqlen, nheads, headdim), dtype),
        dt=_store(np.float32(0.1) * f(batch, seqlen, nheads), dtype),
        dt_bias=np.log(np.expm1(dt_h)).astype(np.float32),
        A=(-np.exp(rng.uniform(0.0, np.log(16.0), size=nheads))).astype(np.float32),
        B=_store(scale * f(batch, seqlen, ngroups, dstate), dtype),
        C=_store(scale * f(batch, seqlen, ngroups, dstate), dtype),
        D=(1.0 + 0.1 * rng.standard_normal(nheads)).astype(np.float32),
    )


def device_scan_inputs(batch: int, dim: int, dstate: int, seqlen: int, seed: int, device):
    """bf16 inputs of one forward pass drawn directly on `device` (for sizes
    whose host-side draw would not fit in host memory): u, z, B, C ~ N(0, 1)
    and delta_raw = 0.1 N(0, 1) from torch's seeded generator on the device,
    rounded to bf16 by torch; A, D (N(1, 0.1)) and the step bias as in
    channel_params.  Returns a dict of device tensors (A, D, delta_bias fp32);
    the oracle reads the rows it checks back from the device."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))

    def draw(shape, scale=1.0):
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if scale != 1.0:
            t.mul_(scale)
        return t.to(torch.bfloat16)

    A, D, bias = channel_params(dim, dstate, "normal", seed)
    return dict(u=draw((batch, dim, seqlen)), delta=draw((batch, dim, seqlen), 0.1),
                z=draw((batch, dim, seqlen)), B=draw((batch, dstate, seqlen)), C=draw((batch, dstate, seqlen)),
                A=torch.from_numpy(A).to(device), D=torch.from_numpy(D).to(device),
                delta_bias=torch.from_numpy(bias).to(device))
