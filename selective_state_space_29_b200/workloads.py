"""Seeded synthetic inputs shaped like the workloads the Mamba pages describe.

This module draws random numbers and nothing else: it holds none of the
scan's arithmetic, so both the CUDA path and the fp64 oracle can take their
inputs from it.  Every tensor is produced by a `torch.Generator` seeded from
(seed, purpose), on whatever device is asked for; the same call on the same
device gives the same bits.

Workloads (one scan or one decode chain each):
  tiny_f32     batch 1, channels 64,   state 16, length 256,        fp32
  mid_bf16     batch 8, channels 3072, state 16, length 2048,       bf16
  large_bf16   batch 4, channels 5120, state 16, length 8192,       bf16 (+ final state)
  long_bf16    batch 1, channels 2048, state 16, length 1,048,576,  bf16, delta in [1e-4, 1e-1]
  decode_bf16  256 sequences x 5120 channels x 16 states, 1000 single-token steps,
               fp32 state, bf16 x / delta / B / C / y
  ssd_mid_bf16 / ssd_long_bf16  the mid and long shapes as Mamba-2 heads of 64
               channels (48 and 32 heads): one scalar A and one step per head
  mimo_mid_bf16  the mid shape with 4 inputs and outputs per channel

Distributions: x ~ N(0,1); delta log-uniform in [lo, hi] (uniform exponent);
B, C ~ N(0,1) per (batch, token, state), shared by all channels; D ~ N(0,1) per
channel; A[d, n] = -(n+1) for the fp32 workload and -(n+1)(1 + 0.1 U_d) with
one U(0,1) per channel otherwise; the decode chain starts from a state drawn
from N(0, 0.1^2) (0.1 is the standard deviation).
"""
from __future__ import annotations

import dataclasses
import math

import torch

_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class ScanWorkload:
    name: str
    batch: int
    length: int
    channels: int
    nstate: int
    dtype: str                 # "f32" or "bf16": dtype of u, delta, B, C and y
    delta_lo: float = 1e-3
    delta_hi: float = 1e-1
    a_mode: str = "channel"    # "s4d" (-(n+1)), "channel" (per-channel scale), "state" (per (d,n) scale)
    final_state: bool = True
    seed: int = 29

    @property
    def torch_dtype(self):
        return _DTYPES[self.dtype]

    @property
    def token_channels(self) -> int:
        return self.batch * self.length * self.channels

    def with_(self, **kw) -> "ScanWorkload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    channels: int
    nstate: int
    steps: int
    dtype: str = "bf16"        # dtype of x, delta, B, C and y; the state is fp32
    delta_lo: float = 1e-3
    delta_hi: float = 1e-1
    a_mode: str = "channel"
    state_std: float = 0.1
    seed: int = 33

    @property
    def torch_dtype(self):
        return _DTYPES[self.dtype]

    @property
    def updates_per_step(self) -> int:
        return self.batch * self.channels

    def with_(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class SsdWorkload:
    """Mamba-2's restricted scan: heads of `headdim` channels, one scalar A
    and one step dt per (batch, token, head)."""
    name: str
    batch: int
    length: int
    heads: int
    headdim: int
    nstate: int
    dtype: str = "bf16"        # dtype of x, dt, B, C and y
    delta_lo: float = 1e-3
    delta_hi: float = 1e-1
    final_state: bool = True
    seed: int = 34

    @property
    def torch_dtype(self):
        return _DTYPES[self.dtype]

    @property
    def channels(self) -> int:
        return self.heads * self.headdim

    @property
    def token_channels(self) -> int:
        return self.batch * self.length * self.channels

    def with_(self, **kw) -> "SsdWorkload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class MimoWorkload:
    """Multi-input multi-output scan: `ranks` inputs and outputs per channel
    sharing one state and one step per (batch, token, channel)."""
    name: str
    batch: int
    length: int
    ranks: int
    channels: int
    nstate: int
    dtype: str = "bf16"
    delta_lo: float = 1e-3
    delta_hi: float = 1e-1
    a_mode: str = "channel"
    seed: int = 36

    @property
    def torch_dtype(self):
        return _DTYPES[self.dtype]

    @property
    def token_channels(self) -> int:
        return self.batch * self.length * self.channels

    def with_(self, **kw) -> "MimoWorkload":
        return dataclasses.replace(self, **kw)


SCAN_WORKLOADS = {
    "tiny_f32": ScanWorkload("tiny_f32", 1, 256, 64, 16, "f32", a_mode="s4d", seed=29),
    "mid_bf16": ScanWorkload("mid_bf16", 8, 2048, 3072, 16, "bf16", seed=30),
    "large_bf16": ScanWorkload("large_bf16", 4, 8192, 5120, 16, "bf16", seed=31),
    "long_bf16": ScanWorkload("long_bf16", 1, 1 << 20, 2048, 16, "bf16", delta_lo=1e-4, seed=32),
}
# the mid and long scan shapes with their channels grouped into heads of 64
SSD_WORKLOADS = {
    "ssd_mid_bf16": SsdWorkload("ssd_mid_bf16", 8, 2048, 48, 64, 16, seed=34),
    "ssd_long_bf16": SsdWorkload("ssd_long_bf16", 1, 1 << 20, 32, 64, 16, delta_lo=1e-4, seed=35),
}
# the mid scan shape with four inputs and outputs per channel (the pages give
# no MIMO sizes; four is a small rank that keeps the state update on FMA)
MIMO_WORKLOADS = {
    "mimo_mid_bf16": MimoWorkload("mimo_mid_bf16", 8, 2048, 4, 3072, 16, seed=36),
}
DECODE_WORKLOADS = {
    "decode_bf16": DecodeWorkload("decode_bf16", 256, 5120, 16, 1000, seed=33),
}


def _gen(device, seed: int, purpose: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(purpose)) & ((1 << 63) - 1))
    return g


def _normal(shape, gen, device, dtype, std=1.0, rows_per_piece=None):
    """N(0, std^2) drawn in fp32 and rounded to `dtype`, in pieces along dim 0
    so that huge tensors never need a full-size fp32 temporary."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(shape[0], -1)
    step = rows_per_piece or max(1, (1 << 27) // max(1, flat.shape[1]))
    for r0 in range(0, shape[0], step):
        piece = torch.randn(flat[r0:r0 + step].shape, generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            piece.mul_(std)
        flat[r0:r0 + step].copy_(piece)
    return out


def _log_uniform(shape, gen, device, dtype, lo, hi):
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(shape[0], -1)
    step = max(1, (1 << 27) // max(1, flat.shape[1]))
    a, b = math.log(lo), math.log(hi)
    for r0 in range(0, shape[0], step):
        piece = torch.rand(flat[r0:r0 + step].shape, generator=gen, device=device, dtype=torch.float32)
        flat[r0:r0 + step].copy_(torch.exp(piece.mul_(b - a).add_(a)))
    return out


def a_matrix(channels: int, nstate: int, mode: str, gen, device) -> torch.Tensor:
    """The fixed, negative-real diagonal A as a (channels, nstate) fp32 array."""
    ramp = torch.arange(1, nstate + 1, device=device, dtype=torch.float32)
    if mode == "s4d":
        return (-ramp).expand(channels, nstate).contiguous()
    if mode == "channel":
        scale = 1.0 + 0.1 * torch.rand((channels, 1), generator=gen, device=device, dtype=torch.float32)
        return (-(ramp * scale)).contiguous()
    if mode == "state":
        scale = 1.0 + 0.1 * torch.rand((channels, nstate), generator=gen, device=device, dtype=torch.float32)
        return (-(ramp * scale)).contiguous()
    if mode == "small":
        # slow decay: |A[d, 0]| log-uniform in [1e-3, 1e-2] per channel, A[d, n] = (n+1) A[d, 0]
        scale = torch.exp(torch.empty((channels, 1), device=device, dtype=torch.float32)
                          .uniform_(math.log(1e-3), math.log(1e-2), generator=gen))
        return (-(ramp * scale)).contiguous()
    if mode == "small_state":
        # slow decay without structure across n: |A[d, n]| log-uniform in [1e-3, 1e-2]
        return (-torch.exp(torch.empty((channels, nstate), device=device, dtype=torch.float32)
                           .uniform_(math.log(1e-3), math.log(1e-2), generator=gen))).contiguous()
    if mode == "random":
        # arbitrary negative values over three decades, no structure across n
        return (-torch.exp(torch.empty((channels, nstate), device=device, dtype=torch.float32)
                           .uniform_(math.log(0.05), math.log(20.0), generator=gen))).contiguous()
    raise ValueError(f"unknown A mode {mode!r}")


def complex_a_imag(channels: int, nstate: int, device) -> torch.Tensor:
    """Rotation rates of a complex diagonal A (imaginary parts), pi * n for
    state n: the pages give none; these are the S4D-Lin imaginary parts, so
    the real parts of the scan workloads' A pair with evenly spaced
    frequencies."""
    return (math.pi * torch.arange(nstate, device=device, dtype=torch.float32)).expand(channels, nstate).contiguous()


def scan_inputs(w: ScanWorkload, device="cpu", seed: int | None = None) -> dict:
    """u, delta (batch, len, channels); B, C (batch, len, nstate) in the
    workload dtype; A (channels, nstate) and D (channels,) in fp32."""
    s = w.seed if seed is None else seed
    dt = w.torch_dtype
    shp_x = (w.batch, w.length, w.channels)
    shp_bc = (w.batch, w.length, w.nstate)
    if w.length == 0 or w.batch == 0:
        u = torch.empty(shp_x, dtype=dt, device=device)
        delta = torch.empty(shp_x, dtype=dt, device=device)
        B = torch.empty(shp_bc, dtype=dt, device=device)
        C = torch.empty(shp_bc, dtype=dt, device=device)
    else:
        u = _normal(shp_x, _gen(device, s, 1), device, dt)
        delta = _log_uniform(shp_x, _gen(device, s, 2), device, dt, w.delta_lo, w.delta_hi)
        B = _normal(shp_bc, _gen(device, s, 3), device, dt)
        C = _normal(shp_bc, _gen(device, s, 4), device, dt)
    A = a_matrix(w.channels, w.nstate, w.a_mode, _gen(device, s, 5), device)
    D = torch.randn((w.channels,), generator=_gen(device, s, 6), device=device, dtype=torch.float32)
    return {"u": u, "delta": delta, "A": A, "B": B, "C": C, "D": D}


def decode_params(w: DecodeWorkload, device="cpu", seed: int | None = None) -> dict:
    """A (channels, nstate), D (channels,) and the initial state
    (batch, channels, nstate), all fp32."""
    s = w.seed if seed is None else seed
    A = a_matrix(w.channels, w.nstate, w.a_mode, _gen(device, s, 5), device)
    D = torch.randn((w.channels,), generator=_gen(device, s, 6), device=device, dtype=torch.float32)
    state = _normal((w.batch, w.channels, w.nstate), _gen(device, s, 7), device, torch.float32,
                    std=w.state_std)
    return {"A": A, "D": D, "state": state}


def decode_step_inputs(w: DecodeWorkload, step: int, device="cpu", seed: int | None = None) -> dict:
    """Fresh x, delta (batch, channels) and B, C (batch, nstate) for one step."""
    s = w.seed if seed is None else seed
    g = _gen(device, s, 1000 + 4 * int(step))
    dt = w.torch_dtype
    x = _normal((w.batch, w.channels), g, device, dt)
    delta = _log_uniform((w.batch, w.channels), g, device, dt, w.delta_lo, w.delta_hi)
    B = _normal((w.batch, w.nstate), g, device, dt)
    C = _normal((w.batch, w.nstate), g, device, dt)
    return {"x": x, "delta": delta, "B": B, "C": C}


def decode_chain_inputs_bulk(w: DecodeWorkload, steps: int, device="cpu", seed: int | None = None) -> dict:
    """`steps` steps of fresh inputs drawn in one go (a different random stream
    from decode_step_inputs, same distributions): x, delta (steps, batch,
    channels); B, C (steps, batch, nstate)."""
    s = w.seed if seed is None else seed
    dt = w.torch_dtype
    return {"x": _normal((steps, w.batch, w.channels), _gen(device, s, 901), device, dt),
            "delta": _log_uniform((steps, w.batch, w.channels), _gen(device, s, 902), device, dt,
                                  w.delta_lo, w.delta_hi),
            "B": _normal((steps, w.batch, w.nstate), _gen(device, s, 903), device, dt),
            "C": _normal((steps, w.batch, w.nstate), _gen(device, s, 904), device, dt)}


def decode_chain_inputs(w: DecodeWorkload, device="cpu", seed: int | None = None) -> dict:
    """All steps' inputs stacked: x, delta (steps, batch, channels); B, C
    (steps, batch, nstate)."""
    steps = [decode_step_inputs(w, i, device, seed) for i in range(w.steps)]
    return {k: torch.stack([st[k] for st in steps]) for k in ("x", "delta", "B", "C")}


def ssd_inputs(w: SsdWorkload, device="cpu", seed: int | None = None) -> dict:
    """x (batch, len, heads*headdim); dt (batch, len, heads); B, C (batch,
    len, nstate) in the workload dtype; A (heads,) and D (channels,) fp32.
    A per head is log-uniform in [-16, -1] (no distribution is given for a
    scalar A; this spans the decay rates of the per-state A of the scan
    workloads, -(n+1) for n < 16)."""
    s = w.seed if seed is None else seed
    dt_ = w.torch_dtype
    shp_x = (w.batch, w.length, w.channels)
    shp_dt = (w.batch, w.length, w.heads)
    shp_bc = (w.batch, w.length, w.nstate)
    if w.length == 0 or w.batch == 0:
        x = torch.empty(shp_x, dtype=dt_, device=device)
        dt = torch.empty(shp_dt, dtype=dt_, device=device)
        B = torch.empty(shp_bc, dtype=dt_, device=device)
        C = torch.empty(shp_bc, dtype=dt_, device=device)
    else:
        x = _normal(shp_x, _gen(device, s, 1), device, dt_)
        dt = _log_uniform(shp_dt, _gen(device, s, 2), device, dt_, w.delta_lo, w.delta_hi)
        B = _normal(shp_bc, _gen(device, s, 3), device, dt_)
        C = _normal(shp_bc, _gen(device, s, 4), device, dt_)
    A = -torch.exp(torch.empty((w.heads,), device=device, dtype=torch.float32)
                   .uniform_(0.0, math.log(16.0), generator=_gen(device, s, 5)))
    D = torch.randn((w.channels,), generator=_gen(device, s, 6), device=device, dtype=torch.float32)
    return {"x": x, "dt": dt, "A": A, "B": B, "C": C, "D": D}


def mimo_inputs(w: MimoWorkload, device="cpu", seed: int | None = None) -> dict:
    """u (batch, len, ranks, channels); delta (batch, len, channels); B, C
    (batch, len, ranks, nstate) in the workload dtype; A (channels, nstate)
    and D (channels,) fp32.  Same distributions as the scan workloads."""
    s = w.seed if seed is None else seed
    dt = w.torch_dtype
    shp_x = (w.batch, w.length, w.ranks, w.channels)
    shp_dl = (w.batch, w.length, w.channels)
    shp_bc = (w.batch, w.length, w.ranks, w.nstate)
    if w.length == 0 or w.batch == 0:
        u = torch.empty(shp_x, dtype=dt, device=device)
        delta = torch.empty(shp_dl, dtype=dt, device=device)
        B = torch.empty(shp_bc, dtype=dt, device=device)
        C = torch.empty(shp_bc, dtype=dt, device=device)
    else:
        u = _normal(shp_x, _gen(device, s, 1), device, dt)
        delta = _log_uniform(shp_dl, _gen(device, s, 2), device, dt, w.delta_lo, w.delta_hi)
        B = _normal(shp_bc, _gen(device, s, 3), device, dt)
        C = _normal(shp_bc, _gen(device, s, 4), device, dt)
    A = a_matrix(w.channels, w.nstate, w.a_mode, _gen(device, s, 5), device)
    D = torch.randn((w.channels,), generator=_gen(device, s, 6), device=device, dtype=torch.float32)
    return {"u": u, "delta": delta, "A": A, "B": B, "C": C, "D": D}
