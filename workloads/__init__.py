"""Seeded synthetic inputs for the selective scan.

This module is the only code that both the CUDA path's tests/bench and the
fp64 oracle consume.  It draws random tensors and nothing else: none of the
scan's arithmetic (discretisation, recurrence, readout, gate) lives here.

The five named workloads are the layer shapes the scan is measured on:
a tiny fp32 case, a Mamba-130M-shaped layer, a Mamba-1.4B-shaped layer, a
long-context scan and an audio-length scan (960 000 samples, the length the
pages use for one second of raw audio).  Draw order per workload is fixed:
u, delta, B, C, z, A-noise, D, delta_bias-uniform.  bf16 workloads draw in
fp32 and round to bf16 (round-to-nearest-even); the oracle is then fed the
same rounded values.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class ScanWorkload:
    name: str
    batch: int
    dim: int
    dstate: int
    seqlen: int
    in_dtype: str          # "f32" or "bf16": u, delta, B, C, z
    has_z: bool            # silu(z) output gate
    a_noise: float         # A[d,n] = -(n+1) * exp(N(0, a_noise)) when > 0
    has_delta_bias: bool   # delta_bias = log(expm1(U[1e-3, 1e-1]))
    has_D: bool = True
    softplus: bool = True

    @property
    def torch_in_dtype(self):
        return torch.float32 if self.in_dtype == "f32" else torch.bfloat16

    @property
    def in_bytes(self) -> int:
        return 4 if self.in_dtype == "f32" else 2

    @property
    def state_updates(self) -> int:
        """B*D*L*N, the count the throughput metric is quoted in."""
        return self.batch * self.dim * self.seqlen * self.dstate

    def algorithmic_bytes(self, out_bytes: int = 4) -> int:
        """Bytes one scan must move: every input read once, y written once.

        u, delta (and z) per (b,d,t); B and C per (b,n,t); A, D and
        delta_bias per channel; y per (b,d,t).  The state never leaves the
        chip, so it adds nothing.
        """
        bdl = self.batch * self.dim * self.seqlen
        row = bdl * (self.in_bytes * (2 + int(self.has_z)) + out_bytes)
        bc = 2 * self.batch * self.dstate * self.seqlen * self.in_bytes
        params = self.dim * self.dstate * 4 + self.dim * 4 * (
            int(self.has_D) + int(self.has_delta_bias))
        return row + bc + params


WORKLOADS = [
    ScanWorkload("tiny-fp32", 1, 16, 4, 256, "f32", has_z=False,
                 a_noise=0.0, has_delta_bias=True),
    ScanWorkload("mamba130m-layer", 8, 1536, 16, 2048, "bf16", has_z=True,
                 a_noise=0.0, has_delta_bias=True),
    ScanWorkload("mamba1.4b-layer", 4, 4096, 16, 4096, "bf16", has_z=True,
                 a_noise=0.1, has_delta_bias=True),
    ScanWorkload("long-context", 1, 1536, 16, 131072, "bf16", has_z=True,
                 a_noise=0.0, has_delta_bias=True),
    ScanWorkload("audio-length", 1, 64, 16, 960000, "f32", has_z=False,
                 a_noise=0.0, has_delta_bias=False),
]
BY_NAME = {w.name: w for w in WORKLOADS}
SEED_BASE = 48000


def seed_of(w: ScanWorkload) -> int:
    return SEED_BASE + WORKLOADS.index(w) if w in WORKLOADS else SEED_BASE + 99


def custom(batch, dim, dstate, seqlen, in_dtype="f32", has_z=True,
           a_noise=0.0, has_delta_bias=True, has_D=True, softplus=True,
           name="custom") -> ScanWorkload:
    return ScanWorkload(name, batch, dim, dstate, seqlen, in_dtype, has_z,
                        a_noise, has_delta_bias, has_D, softplus)


def make_inputs(w: ScanWorkload, seed: int | None = None,
                device: str | torch.device = "cpu") -> dict:
    """Draw the inputs of workload ``w`` with a seeded torch generator.

    Returns a dict of tensors on ``device``: u, delta, z (batch, dim, L) and
    B, C (batch, N, L) in the workload's input dtype; A (dim, N), D (dim,),
    delta_bias (dim,) in fp32 (None where the workload has none).
    """
    seed = seed_of(w) if seed is None else seed
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    f32 = torch.float32
    dt = w.torch_in_dtype

    def normal(*shape, std=1.0):
        x = torch.randn(*shape, generator=g, device=dev, dtype=f32)
        return x if std == 1.0 else x * std

    row = (w.batch, w.dim, w.seqlen)
    u = normal(*row).to(dt)
    delta = normal(*row).to(dt)
    B = normal(w.batch, w.dstate, w.seqlen).to(dt)
    C = normal(w.batch, w.dstate, w.seqlen).to(dt)
    z = normal(*row).to(dt) if w.has_z else None
    base = -torch.arange(1, w.dstate + 1, device=dev, dtype=f32)
    A = base.expand(w.dim, w.dstate).contiguous()
    if w.a_noise > 0:
        A = A * torch.exp(normal(w.dim, w.dstate, std=w.a_noise))
    D = normal(w.dim) if w.has_D else None
    if w.has_delta_bias:
        v = torch.rand(w.dim, generator=g, device=dev, dtype=torch.float64)
        v = 1e-3 + (1e-1 - 1e-3) * v
        # inverse of softplus: the bias that makes softplus(bias) == v
        delta_bias = torch.log(torch.expm1(v)).to(f32)
    else:
        delta_bias = None
    return dict(u=u, delta=delta, A=A, B=B, C=C, D=D, z=z,
                delta_bias=delta_bias)


def to_numpy_f64(inputs: dict) -> dict:
    """The same values widened to float64 on the host (for the oracle)."""
    out = {}
    for k, v in inputs.items():
        out[k] = None if v is None else v.detach().to("cpu", torch.float64).numpy()
    return out


def describe(w: ScanWorkload) -> str:
    return (f"{w.name}: batch={w.batch} D={w.dim} N={w.dstate} L={w.seqlen} "
            f"{w.in_dtype}{' +z' if w.has_z else ''}")


# --------------------------------------------------------------------------
# Mamba-2 (SSD) inputs: A is one scalar per head.  Shapes follow a Mamba-2
# layer: heads of 64 channels, 128 states (eight times Mamba-1's 16), one
# group of B, C shared by all heads.  Draw order: x, dt, B, C, z, A, D,
# dt_bias, h0.  A[h] = -U[1, 16]; dt_bias as delta_bias above; x, dt, B,
# C, z ~ N(0, 1) rounded to bf16; D ~ N(0, 1); h0 ~ N(0, 1) / 4.


@dataclasses.dataclass(frozen=True)
class SsdWorkload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int = 64
    ngroups: int = 1
    dstate: int = 128
    has_z: bool = False
    has_D: bool = True
    has_dt_bias: bool = True
    softplus: bool = True

    def algorithmic_bytes(self, out_bytes: int = 4) -> int:
        """x (and z) read and y written once per (b, t, h, p); dt once per
        (b, t, h); B and C once per (b, t, g, n); A, D, dt_bias per head."""
        btp = self.batch * self.seqlen * self.nheads * self.headdim
        row = btp * (2 * (1 + int(self.has_z)) + out_bytes)
        dt = self.batch * self.seqlen * self.nheads * 2
        bc = 2 * self.batch * self.seqlen * self.ngroups * self.dstate * 2
        return row + dt + bc + self.nheads * 4 * (1 + int(self.has_D) + int(self.has_dt_bias))

    def chunk_flops(self, chunk: int = 128) -> int:
        """Matrix-product FLOPs of the chunked form per full pass: per chunk
        and group the scores C B^T (2 Q^2 N, shared by the group's heads);
        per chunk and head the masked product with X (2 Q^2 P), the
        carried-state readout C h (2 Q N P) and the chunk's state update
        B^T X (2 Q N P)."""
        Q, N, P = chunk, self.dstate, self.headdim
        nch = -(-self.seqlen // chunk)
        scores = self.batch * self.ngroups * nch * 2 * Q * Q * N
        return scores + self.batch * self.nheads * nch * (2 * Q * Q * P + 4 * Q * N * P)


SSD_WORKLOADS = [
    SsdWorkload("ssd-small", 2, 300, 4, ngroups=2, has_z=True),
    SsdWorkload("mamba2-2.7b-layer", 8, 2048, 80),
]
SSD_BY_NAME = {w.name: w for w in SSD_WORKLOADS}


def make_ssd_inputs(w: SsdWorkload, seed: int, device: str | torch.device = "cpu",
                    h0: bool = False) -> dict:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    f32, bf = torch.float32, torch.bfloat16

    def normal(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=f32)

    bl = (w.batch, w.seqlen)
    x = normal(*bl, w.nheads, w.headdim).to(bf)
    dt = normal(*bl, w.nheads).to(bf)
    B = normal(*bl, w.ngroups, w.dstate).to(bf)
    C = normal(*bl, w.ngroups, w.dstate).to(bf)
    z = normal(*bl, w.nheads, w.headdim).to(bf) if w.has_z else None
    A = -(1.0 + 15.0 * torch.rand(w.nheads, generator=g, device=dev, dtype=f32))
    D = normal(w.nheads) if w.has_D else None
    if w.has_dt_bias:
        v = torch.rand(w.nheads, generator=g, device=dev, dtype=torch.float64)
        v = 1e-3 + (1e-1 - 1e-3) * v
        dt_bias = torch.log(torch.expm1(v)).to(f32)
    else:
        dt_bias = None
    hz = normal(w.batch, w.nheads, w.headdim, w.dstate) * 0.25 if h0 else None
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D, z=z, dt_bias=dt_bias, h0=hz)


__all__ = ["ScanWorkload", "WORKLOADS", "BY_NAME", "custom", "make_inputs",
           "to_numpy_f64", "seed_of", "describe", "SsdWorkload", "SSD_WORKLOADS",
           "SSD_BY_NAME", "make_ssd_inputs"]
