"""Seeded synthetic inputs for the selective-scan workloads.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the scan's arithmetic, and it imports neither the oracle nor
the CUDA library: both sides receive the very same stored arrays from here.

Shapes follow the layer sizes of the Mamba models the pages discuss (a tiny
fp32 case, Mamba-130M and Mamba-2.8B mixer layers with expand 2, a 131072-token
sequence, and a 256-sequence decode batch).  The pages use no public dataset
for this path; every input is synthetic.

Recipe (per config, ``numpy.random.default_rng(seed)``, seed = config index by
default, draws in float32 in this order):
  x, z ~ N(0, 1) and delta_raw ~ N(0, 0.1^2), each [batch][dim][seqlen];
  B, C ~ N(0, 1), each [batch][dstate][seqlen];
  dt0[d] = exp(U[ln lo, ln hi]) (float64), delta_bias = log(expm1(dt0))
  (the inverse of softplus, so softplus(bias) = dt0);
  h0 ~ N(0, 1) [batch][dim][dstate] when the config has an initial state.
  A[d, n] = -(n + 1) (S4D-real), D = 1, float32.
Activations are rounded to bfloat16 (round to nearest even) from float32 for
the bf16 workloads and kept as float32 for the tiny fp32 one.  bfloat16 arrays are carried
as uint16 bit patterns.

The decode config draws each step's tokens from its own stream
``SeedSequence([seed, phase, step])`` (phase 0: the 64 prefill steps, phase 1:
the decode steps), so that any step can be regenerated on its own.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

_CHUNK = 1 << 24  # elements per draw call (bounds host temporaries)


@dataclass(frozen=True)
class Config:
    index: int
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    dtype: str  # "f32" or "bf16"
    has_h0: bool = False
    dt_range: tuple = (1e-3, 1e-1)
    decode_steps: int = 0
    prefill_steps: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def channels(self) -> int:
        return self.batch * self.dim


CONFIGS = {
    0: Config(0, "tiny-fp32 1x256x64", 1, 256, 64, 16, "f32"),
    1: Config(1, "mamba-130m-layer 8x2048x1536", 8, 2048, 1536, 16, "bf16"),
    2: Config(2, "mamba-2.8b-layer 4x4096x5120", 4, 4096, 5120, 16, "bf16"),
    3: Config(3, "long-seq 1x131072x2048 h0", 1, 131072, 2048, 16, "bf16", has_h0=True,
              dt_range=(1e-4, 1e-1)),
    4: Config(4, "decode 256x5120 N16 x1024 steps", 256, 1, 5120, 16, "bf16",
              decode_steps=1024, prefill_steps=64),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def _normal(rng, shape, scale, dtype):
    """N(0, scale^2) of the given shape, drawn in float32 chunks, stored as dtype."""
    n = int(np.prod(shape))
    if dtype == "f32":
        out = np.empty(n, np.float32)
    else:
        out = np.empty(n, np.uint16)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        v = rng.standard_normal(e - s, dtype=np.float32)
        if scale != 1.0:
            v *= np.float32(scale)
        out[s:e] = v if dtype == "f32" else f32_to_bf16_bits(v)
    return out.reshape(shape)


def _params(rng, cfg_dim, dstate, dt_range):
    lo, hi = dt_range
    dt0 = np.exp(rng.uniform(np.log(lo), np.log(hi), size=cfg_dim))
    delta_bias = np.log(np.expm1(dt0)).astype(np.float32)
    A = np.tile(-(np.arange(dstate, dtype=np.float32) + 1.0), (cfg_dim, 1))
    D = np.ones(cfg_dim, np.float32)
    return A, D, delta_bias


def make_inputs(cfg: Config | int, seed: int | None = None, seqlen: int | None = None) -> dict:
    """Inputs of a forward-scan config.  `seqlen` may shorten the sequence
    (same distributions) for quick checks."""
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    seed = cfg.index if seed is None else seed
    L = cfg.seqlen if seqlen is None else seqlen
    rng = np.random.default_rng(seed)
    b, d, n = cfg.batch, cfg.dim, cfg.dstate
    x = _normal(rng, (b, d, L), 1.0, cfg.dtype)
    delta = _normal(rng, (b, d, L), 0.1, cfg.dtype)
    z = _normal(rng, (b, d, L), 1.0, cfg.dtype)
    B = _normal(rng, (b, n, L), 1.0, cfg.dtype)
    C = _normal(rng, (b, n, L), 1.0, cfg.dtype)
    A, D, delta_bias = _params(rng, d, n, cfg.dt_range)
    h0 = rng.standard_normal((b, d, n), dtype=np.float32) if cfg.has_h0 else None
    return dict(x=x, delta=delta, z=z, B=B, C=C, A=A, D=D, delta_bias=delta_bias, h0=h0,
                softplus=True)


def custom_inputs(batch, seqlen, dim, dstate, dtype="bf16", seed=0, has_h0=False,
                  dt_range=(1e-3, 1e-1), delta_scale=0.1) -> dict:
    """Inputs of any shape with the configs' distributions (for edge cases)."""
    rng = np.random.default_rng(seed)
    x = _normal(rng, (batch, dim, seqlen), 1.0, dtype)
    delta = _normal(rng, (batch, dim, seqlen), delta_scale, dtype)
    z = _normal(rng, (batch, dim, seqlen), 1.0, dtype)
    B = _normal(rng, (batch, dstate, seqlen), 1.0, dtype)
    C = _normal(rng, (batch, dstate, seqlen), 1.0, dtype)
    A, D, delta_bias = _params(rng, dim, dstate, dt_range)
    h0 = rng.standard_normal((batch, dim, dstate), dtype=np.float32) if has_h0 else None
    return dict(x=x, delta=delta, z=z, B=B, C=C, A=A, D=D, delta_bias=delta_bias, h0=h0,
                softplus=True)


def decode_params(cfg: Config | int = 4, seed: int | None = None) -> dict:
    """A, D, delta_bias of the decode config."""
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    seed = cfg.index if seed is None else seed
    rng = np.random.default_rng(np.random.SeedSequence([seed, 2, 0]))
    A, D, delta_bias = _params(rng, cfg.dim, cfg.dstate, cfg.dt_range)
    return dict(A=A, D=D, delta_bias=delta_bias, softplus=True)


def decode_tokens(cfg: Config | int, step: int, phase: int = 1, seed: int | None = None,
                  batch: int | None = None) -> dict:
    """One token per sequence for decode step `step` (phase 0 = prefill).

    x, delta, z: [batch][dim]; B, C: [batch][dstate]."""
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    seed = cfg.index if seed is None else seed
    b = cfg.batch if batch is None else batch
    rng = np.random.default_rng(np.random.SeedSequence([seed, phase, step]))
    x = _normal(rng, (b, cfg.dim), 1.0, cfg.dtype)
    delta = _normal(rng, (b, cfg.dim), 0.1, cfg.dtype)
    z = _normal(rng, (b, cfg.dim), 1.0, cfg.dtype)
    B = _normal(rng, (b, cfg.dstate), 1.0, cfg.dtype)
    C = _normal(rng, (b, cfg.dstate), 1.0, cfg.dtype)
    return dict(x=x, delta=delta, z=z, B=B, C=C)


def compulsory_bytes_fwd(batch, seqlen, dim, dstate, act_bytes, has_h0, write_h_last,
                         has_z=True, has_D=True, has_bias=True):
    """Bytes a forward scan must move at least once: read x, delta, z, B, C,
    A, D, bias, h0 (if given); write out and h_last (if requested)."""
    tok = batch * dim * seqlen
    rd = tok * act_bytes * (2 + (1 if has_z else 0))
    rd += 2 * batch * dstate * seqlen * act_bytes
    rd += dim * dstate * 4 + (dim * 4 if has_D else 0) + (dim * 4 if has_bias else 0)
    if has_h0:
        rd += batch * dim * dstate * 4
    wr = tok * act_bytes + (batch * dim * dstate * 4 if write_h_last else 0)
    return rd + wr


def compulsory_bytes_step(batch, dim, dstate, act_bytes):
    """Bytes a decode step must move: the fp32 state read and written, the
    token tensors read, out written, and the parameters read."""
    state = 2 * batch * dim * dstate * 4
    tok = batch * dim * act_bytes * 4 + 2 * batch * dstate * act_bytes
    params = dim * dstate * 4 + 2 * dim * 4
    return state + tok + params
