"""Seeded synthetic inputs and the named workloads of the SSD layer.

This module only draws random numbers and rounds them to the I/O dtype; it
holds none of the SSD arithmetic. Both the CUDA path and the CPU oracle
consume the buffers it returns, so the two always see identical inputs.

Recipe (one numpy PCG64 sub-stream per tensor, ``SeedSequence(seed).spawn(6)``
in the order x, dt, A, Bm, Cm, D; everything drawn in fp64, then rounded once,
round-to-nearest-even, to the tensor's storage dtype):

* x ~ N(0, 1)                                  [B, L, H, P], I/O dtype
* dt = exp(U[ln 1e-3, ln 1e-1])                [B, L, H], fp32 (the step size after
  the softplus of the selection mechanism; "Mamba paper review", section 3.1)
* A_h = -exp(U[0, ln 16])                      [H], fp32 (A < 0)
* Bm, Cm ~ N(0, 1) / sqrt(N)                   [B, L, G, N], I/O dtype
* D ~ N(0, 1)                                  [H], fp32

Special cases replace dt and A (the oracle pins of the same names):
``linear_attention`` (dt = 1, A = 0, so a_t = 1), ``retnet`` (dt = 1,
A = ln 0.99, so a_t = 0.99) and ``zero_decay`` (dt = 0.1, A = -1e4, so
a_t = exp(-1000) = 0 in fp32 and fp64).

bf16 tensors are returned as their raw uint16 bit patterns.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

IO_DTYPES = ("f32", "bf16")


def round_to_bf16_bits(a64: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (8 significant bits, RNE); return uint16 bits.
    Values are finite and far from the bf16 subnormal range in every recipe here."""
    a64 = np.ascontiguousarray(a64, dtype=np.float64)
    bits = a64.view(np.uint64)
    # keep 7 explicit mantissa bits of the 52: round at bit 45, ties to even
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    rounded = (bits + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f32 = rounded.view(np.float64).astype(np.float32)  # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Upcast a stored tensor (fp32, or bf16 bits) to fp64 exactly."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _store(a64: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16_bits(a64)
    if dtype == "f32":
        return a64.astype(np.float32)
    raise ValueError(f"unknown I/O dtype {dtype!r}")


@dataclasses.dataclass
class SSDInputs:
    """Host buffers of one forward call; x, Bm, Cm in the I/O dtype."""
    dtype: str
    x: np.ndarray    # [B, L, H, P]
    dt: np.ndarray   # [B, L, H] fp32
    A: np.ndarray    # [H] fp32
    Bm: np.ndarray   # [B, L, G, N]
    Cm: np.ndarray   # [B, L, G, N]
    D: np.ndarray    # [H] fp32

    @property
    def shape(self):
        Bsz, L, H, P = self.x.shape
        return Bsz, L, H, P, self.Bm.shape[2], self.Bm.shape[3]

    def f64(self, b0: int = 0, b1: int | None = None, heads=None):
        """fp64 copies for the oracle, optionally of batches [b0, b1) and a
        contiguous head range ``heads = (h0, h1)`` whose groups are kept whole
        (the caller passes a head range aligned to groups, or G == 1)."""
        b1 = self.x.shape[0] if b1 is None else b1
        Bsz, L, H, P, G, N = self.shape
        h0, h1 = (0, H) if heads is None else heads
        hpg = H // G
        g0, g1 = h0 // hpg, (h1 - 1) // hpg + 1
        if heads is not None and G > 1 and (h0 % hpg or h1 % hpg):
            raise ValueError("head range must be aligned to groups when G > 1")
        x = to_f64(self.x[b0:b1, :, h0:h1], self.dtype)
        Bm = to_f64(self.Bm[b0:b1, :, g0:g1], self.dtype)
        Cm = to_f64(self.Cm[b0:b1, :, g0:g1], self.dtype)
        dt = self.dt[b0:b1, :, h0:h1].astype(np.float64)
        A = self.A[h0:h1].astype(np.float64)
        D = self.D[h0:h1].astype(np.float64)
        return x, dt, A, Bm, Cm, D


def make_inputs(Bsz, L, H, P, G, N, dtype="bf16", seed=0, kind="random") -> SSDInputs:
    if H % G:
        raise ValueError("H must be a multiple of G")
    s_x, s_dt, s_A, s_B, s_C, s_D = (np.random.Generator(np.random.PCG64(s))
                                     for s in np.random.SeedSequence(seed).spawn(6))
    x = _store(s_x.standard_normal((Bsz, L, H, P)), dtype)
    dt64 = np.exp(s_dt.uniform(math.log(1e-3), math.log(1e-1), (Bsz, L, H)))
    A64 = -np.exp(s_A.uniform(0.0, math.log(16.0), (H,)))
    scale = 1.0 / math.sqrt(N)
    Bm = _store(s_B.standard_normal((Bsz, L, G, N)) * scale, dtype)
    Cm = _store(s_C.standard_normal((Bsz, L, G, N)) * scale, dtype)
    D64 = s_D.standard_normal((H,))
    if kind == "linear_attention":
        dt64 = np.ones_like(dt64)
        A64 = np.zeros_like(A64)
    elif kind == "retnet":
        dt64 = np.ones_like(dt64)
        A64 = np.full_like(A64, math.log(0.99))
    elif kind == "zero_decay":
        dt64 = np.full_like(dt64, 0.1)
        A64 = np.full_like(A64, -1.0e4)
    elif kind == "mixed_decay":
        # heads 1 mod 3 decay by 2^-70 .. 2^-700 per token, heads 2 mod 3 have
        # a zero step every 37th token, the rest are drawn as above
        strong = -np.exp(s_A.uniform(math.log(500.0), math.log(5000.0), (H,)))
        A64 = np.where(np.arange(H) % 3 == 1, strong, A64)
        gaps = (np.arange(L)[None, :, None] % 37 == 5) & (np.arange(H)[None, None, :] % 3 == 2)
        dt64 = np.where(gaps, 0.0, dt64)
    elif kind != "random":
        raise ValueError(f"unknown input kind {kind!r}")
    return SSDInputs(dtype, x, dt64.astype(np.float32), A64.astype(np.float32), Bm, Cm,
                     D64.astype(np.float32))


@dataclasses.dataclass
class StepInputs:
    """Host buffers of one decode step; x, Bm, Cm in the I/O dtype."""
    dtype: str
    x: np.ndarray      # [B, H, P]
    dt: np.ndarray     # [B, H] fp32
    A: np.ndarray      # [H] fp32
    Bm: np.ndarray     # [B, G, N]
    Cm: np.ndarray     # [B, G, N]
    D: np.ndarray      # [H] fp32
    state: np.ndarray  # [B, H, P, N] fp32


def make_step_inputs(Bsz, H, P, G, N, dtype="bf16", seed=0) -> StepInputs:
    """Same distributions as ``make_inputs`` for one token, plus a random fp32
    state ~ N(0, 1) drawn from a seventh sub-stream."""
    streams = [np.random.Generator(np.random.PCG64(s))
               for s in np.random.SeedSequence(seed).spawn(7)]
    s_x, s_dt, s_A, s_B, s_C, s_D, s_h = streams
    scale = 1.0 / math.sqrt(N)
    return StepInputs(
        dtype,
        _store(s_x.standard_normal((Bsz, H, P)), dtype),
        np.exp(s_dt.uniform(math.log(1e-3), math.log(1e-1), (Bsz, H))).astype(np.float32),
        (-np.exp(s_A.uniform(0.0, math.log(16.0), (H,)))).astype(np.float32),
        _store(s_B.standard_normal((Bsz, G, N)) * scale, dtype),
        _store(s_C.standard_normal((Bsz, G, N)) * scale, dtype),
        s_D.standard_normal((H,)).astype(np.float32),
        s_h.standard_normal((Bsz, H, P, N)).astype(np.float32),
    )


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    H: int
    P: int
    G: int
    N: int
    chunk: int
    dtype: str
    kind: str = "random"

    @property
    def tokens(self) -> int:
        return self.B * self.L

    def make(self, seed: int = 0) -> SSDInputs:
        return make_inputs(self.B, self.L, self.H, self.P, self.G, self.N, self.dtype, seed,
                           self.kind)


TINY_F32 = Workload("tiny-fp32 B1 L64 H2 P8 N8 G1 Q16", 1, 64, 2, 8, 1, 8, 16, "f32")
LAYER_370M = Workload("mamba2-370m-layer-bf16 B8 L2048 H32 P64 N128 G1 Q256",
                      8, 2048, 32, 64, 1, 128, 256, "bf16")
LAYER_2P7B = Workload("mamba2-2.7b-layer-bf16 B4 L4096 H80 P64 N128 G1 Q256",
                      4, 4096, 80, 64, 1, 128, 256, "bf16")
LONG_CONTEXT = Workload("long-context-bf16 B1 L65536 H32 P64 N128 G1 Q256",
                        1, 65536, 32, 64, 1, 128, 256, "bf16")
DECODE = dict(name="decode-step-bf16 B64 H32 P64 N128 G1", B=64, H=32, P=64, G=1, N=128,
              dtype="bf16")


def sweep_workloads(kinds=("random",)):
    """State-size / grouping sweep: B2 L8192 H64 P64 G8, N in 16..256, Q in {128, 256}."""
    out = []
    for kind in kinds:
        for N in (16, 32, 64, 128, 256):
            for Q in (128, 256):
                tag = "" if kind == "random" else f" {kind}"
                out.append(Workload(f"sweep-bf16 B2 L8192 H64 P64 G8 N{N} Q{Q}{tag}",
                                    2, 8192, 64, 64, 8, N, Q, "bf16", kind))
    return out
