"""Seeded synthetic inputs for multi-scale retention.

This module holds the input recipe only: sizes, random draws and the
rounding of draws to the storage dtype.  It contains none of the retention
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it without sharing any of the method.

Recipe (the same for every workload):
  * numpy PCG64 generator seeded with the workload's seed;
  * q, k, v drawn i.i.d. from N(0, 1), in that order, each scaled by
    1/sqrt(d_k), cast to float32 and, for bf16 workloads, rounded to bf16
    with round-to-nearest-even;
  * per-head decays gamma_h = 1 - 2^(-5-h), h = 0..H-1 (the multi-scale
    schedule of "RetNet - Retentive Network - A Successor to Transformer for
    LLMs", section Methods / Multi-Scale Retention), stored as float32
    (exact for h <= 18);
  * the optional initial state is drawn after q, k, v from N(0, 1) scaled by
    1/sqrt(d_k), float32.

The consumer gets the stored values twice: as the raw storage array (float32,
or uint16 bf16 bit patterns) for the device, and as float64 for the oracle.
Both views hold exactly the same numbers.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    dk: int
    dv: int
    dtype: str          # "f32" or "bf16"
    chunk: int          # chunk size of the chunkwise form
    gn_eps: float       # < 0: no GroupNorm
    state_out: bool     # whether the final state is requested
    seed: int

    @property
    def tokens(self) -> int:
        return self.B * self.N


# The five workloads the hot path is measured and checked on.  Shapes follow
# the pages' setting (8k context, batch 8, 6.7B-class head layout).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 4, 256, 64, 64, "f32", 64, -1.0, True, 1),
    "l1p3b_bf16": Workload("l1p3b_bf16", 8, 8, 2048, 256, 256, "bf16", 128, -1.0, False, 2),
    "l6p7b_8k_bf16": Workload("l6p7b_8k_bf16", 8, 16, 8192, 256, 512, "bf16", 512, 1e-5, False, 3),
    # decode: prefill length N, then DECODE_STEPS single-token steps
    "decode_6p7b": Workload("decode_6p7b", 8, 16, 8192, 256, 512, "bf16", 512, -1.0, True, 4),
    "long_64k_bf16": Workload("long_64k_bf16", 1, 16, 65536, 256, 512, "bf16", 512, -1.0, True, 5),
}
DECODE_STEPS = 1024


def msr_gammas(H: int) -> np.ndarray:
    """gamma_h = 1 - 2^(-5-h) for h = 0..H-1, float32."""
    return np.array([1.0 - 2.0 ** (-5 - h) for h in range(H)], dtype=np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    r = ((u + bias) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@dataclasses.dataclass
class Tensor:
    """One input: `store` is what goes to the device, `exact` the same values in float64."""
    store: np.ndarray
    exact: np.ndarray
    dtype: str


def _as_dtype(x32: np.ndarray, dtype: str) -> Tensor:
    if dtype == "f32":
        return Tensor(x32, x32.astype(np.float64), "f32")
    if dtype == "bf16":
        bits = f32_to_bf16_bits(x32)
        return Tensor(bits, bf16_bits_to_f64(bits), "bf16")
    raise ValueError(dtype)


def from_values(x, dtype: str) -> Tensor:
    """A Tensor holding the given values, cast to float32 (and for bf16
    rounded to nearest even)."""
    return _as_dtype(np.asarray(x, dtype=np.float32), dtype)


def draw(rng: np.random.Generator, shape, scale: float, dtype: str) -> Tensor:
    x = (rng.standard_normal(size=shape) * scale).astype(np.float32)
    return _as_dtype(x, dtype)


def make_inputs(B, H, N, dk, dv, dtype="bf16", seed=0, with_state=False, scale=None,
                gammas=None):
    """q, k, v (and optionally an initial state) for one retention call.

    Returns a dict with Tensor entries q, k, v, state (or None) and the
    float32 gamma array.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    s = (1.0 / math.sqrt(dk)) if scale is None else scale
    q = draw(rng, (B, H, N, dk), s, dtype)
    k = draw(rng, (B, H, N, dk), s, dtype)
    v = draw(rng, (B, H, N, dv), s, dtype)
    st = draw(rng, (B, H, dk, dv), s, "f32") if with_state else None
    g = msr_gammas(H) if gammas is None else np.asarray(gammas, dtype=np.float32)
    return {"q": q, "k": k, "v": v, "state": st, "gammas": g}


def rotation_angles(d: int, seed: int = 0) -> np.ndarray:
    """Angles (radians per position) for the d/2 channel pairs of the xPos
    rotation: the pages give no values, so a geometric spread from 1 down to
    1e-4, shuffled with the seed so that a mix-up of pairs changes the result."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.permutation(np.geomspace(1.0, 1e-4, d // 2)).astype(np.float32)


def make_head_inputs(w: Workload, b: int, h: int, N: int | None = None):
    """Inputs of one (batch, head) pair of a workload, drawn independently of
    the others, so that a sampled head can be rebuilt without drawing the
    whole batch.  Seeded by (workload seed, b, h)."""
    n = w.N if N is None else N
    rng = np.random.Generator(np.random.PCG64([w.seed, b, h]))
    s = 1.0 / math.sqrt(w.dk)
    q = draw(rng, (n, w.dk), s, w.dtype)
    k = draw(rng, (n, w.dk), s, w.dtype)
    v = draw(rng, (n, w.dv), s, w.dtype)
    return q, k, v


def make_decode_token(w: Workload, step: int):
    """q, k, v of one decode step for all (batch, head) pairs: [B,H,d]."""
    rng = np.random.Generator(np.random.PCG64([w.seed, 1_000_000 + step]))
    s = 1.0 / math.sqrt(w.dk)
    q = draw(rng, (w.B, w.H, w.dk), s, w.dtype)
    k = draw(rng, (w.B, w.H, w.dk), s, w.dtype)
    v = draw(rng, (w.B, w.H, w.dv), s, w.dtype)
    return q, k, v


def to_torch(t: Tensor, device="cuda", pin=False):
    """Move a stored input to torch without changing a bit: float32 stays
    float32, bf16 bit patterns become torch.bfloat16."""
    import torch
    if t.dtype == "f32":
        x = torch.from_numpy(np.ascontiguousarray(t.store))
    else:
        x = torch.from_numpy(np.ascontiguousarray(t.store).view(np.int16)).view(torch.bfloat16)
    if pin:
        return x.pin_memory()
    return x.to(device)


def from_torch(x) -> np.ndarray:
    """A torch tensor (any device, float32 or bf16) as float64 numpy."""
    import torch
    return x.detach().to(device="cpu", dtype=torch.float64).numpy()
