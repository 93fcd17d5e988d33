"""Seeded synthetic inputs for the WKV kernels and for the fp64 oracle.

This module draws random numbers and rounds them to the storage types the
kernels read. It holds none of the WKV arithmetic: every value it returns is an
*input* (the decay rate w is drawn as exp(time_decay) because that is how the
RWKV-4 model parameterises it, see ``RWKV_TimeMix.__init__`` on the
"代码连连看——RWKV" RWKV-LM v4 walkthrough page, the fancy time_decay init;
the RWKV-6 decay is drawn as exp(-exp(d)) so that it lies in (0, 1)).

Both the CUDA path (through the binding) and the oracle (through the tests and
the bench's CPU baseline) consume exactly the arrays returned here, so they see
the same rounded numbers: bf16 tensors are returned as their raw uint16 bit
patterns plus an exact float32 decoding.

Draw order per generator is fixed (numpy PCG64, one stream per call):
  RWKV-4: time_decay[C], u[C], k[B,T,C], v[B,T,C], gy[B,T,C]
  RWKV-6: d[B,T,H*K], u[H*K], r, k, v  (each [B,T,H*K])
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "Wkv4Recipe",
    "gate_input",
    "Wkv6Recipe",
    "wkv4_inputs",
    "wkv4_slot_inputs",
    "wkv6_inputs",
    "WKV4_RECIPES",
    "WKV6_RECIPES",
    "Wkv7Recipe",
    "WKV7_RECIPES",
    "wkv7_inputs",
    "feed_schedule",
]


# ----------------------------------------------------------------------------
# bf16 storage helpers (bit manipulation only)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the uint16 bit patterns. Inputs must be finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # RNE: add 0x7FFF plus the lsb of the kept half, then truncate.
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact decoding of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(x32: np.ndarray, dtype: str):
    """Return (storage array, exact float32 view of what is stored)."""
    if dtype == "f32":
        x32 = np.ascontiguousarray(x32, dtype=np.float32)
        return x32, x32
    if dtype == "bf16":
        bits = f32_to_bf16_bits(x32)
        return bits, bf16_bits_to_f32(bits)
    raise ValueError(f"unknown dtype {dtype!r}")


# ----------------------------------------------------------------------------
# RWKV-4 recipes
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Wkv4Recipe:
    """Shape and value distributions of one RWKV-4 WKV workload."""

    name: str
    B: int
    T: int
    C: int
    dtype: str                 # storage type of k, v, y, gy, gk, gv: "f32" | "bf16"
    td_lo: float               # time_decay ~ U(td_lo, td_hi); w = exp(time_decay)
    td_hi: float
    u_lo: float                # u (time_first) ~ U(u_lo, u_hi)
    u_hi: float
    k_std: float               # k ~ N(0, k_std^2)
    v_std: float = 1.0         # v ~ N(0, v_std^2)
    backward: bool = False     # draw gy ~ N(0, 1) too

    def with_shape(self, B=None, T=None, C=None, name=None):
        return dataclasses.replace(
            self, B=self.B if B is None else B, T=self.T if T is None else T,
            C=self.C if C is None else C, name=name or self.name)


WKV4_RECIPES = {
    # forward only, fp32, small enough for the oracle in well under a second
    "wkv4_fwd_f32_small": Wkv4Recipe("wkv4_fwd_f32_small", 2, 64, 128, "f32",
                                     -6.0, 1.0, -1.0, 1.0, 1.0),
    # forward+backward, fp32, RWKV-4 169M width; k wide to stress the running max
    "wkv4_fb_f32_169m": Wkv4Recipe("wkv4_fb_f32_169m", 8, 1024, 768, "f32",
                                   -6.0, 1.0, -1.0, 1.0, 2.0, backward=True),
    # forward+backward, bf16 I/O, RWKV-4 3B width
    "wkv4_fb_bf16_3b": Wkv4Recipe("wkv4_fb_bf16_3b", 16, 4096, 2560, "bf16",
                                  -8.0, 2.0, -2.0, 2.0, 1.5, backward=True),
    # roofline shapes at C=4096 with the 3B-width distributions
    "wkv4_fb_f32_c4096": Wkv4Recipe("wkv4_fb_f32_c4096", 16, 4096, 4096, "f32",
                                    -8.0, 2.0, -2.0, 2.0, 1.5, backward=True),
    "wkv4_fb_bf16_c4096": Wkv4Recipe("wkv4_fb_bf16_c4096", 16, 4096, 4096, "bf16",
                                     -8.0, 2.0, -2.0, 2.0, 1.5, backward=True),
}


def wkv4_inputs(recipe: Wkv4Recipe, seed: int = 0) -> dict:
    """Draw one RWKV-4 workload.

    Returns a dict with
      w, u        float32 [C]   (w = exp(time_decay) > 0)
      time_decay  float32 [C]
      k, v        storage arrays [B,T,C] (float32, or uint16 bf16 bits)
      k32, v32    exact float32 values of k, v
      gy, gy32    (only when recipe.backward) same for the upstream gradient
    """
    B, T, C = recipe.B, recipe.T, recipe.C
    rng = np.random.Generator(np.random.PCG64(seed))
    td = rng.uniform(recipe.td_lo, recipe.td_hi, size=C)             # fp64
    u = rng.uniform(recipe.u_lo, recipe.u_hi, size=C).astype(np.float32)
    k = rng.standard_normal(size=(B, T, C), dtype=np.float32)
    if recipe.k_std != 1.0:
        k *= np.float32(recipe.k_std)
    v = rng.standard_normal(size=(B, T, C), dtype=np.float32)
    if recipe.v_std != 1.0:
        v *= np.float32(recipe.v_std)
    out = {
        "time_decay": td.astype(np.float32),
        "w": np.exp(td).astype(np.float32),
        "u": u,
    }
    out["k"], out["k32"] = _store(k, recipe.dtype)
    del k
    out["v"], out["v32"] = _store(v, recipe.dtype)
    del v
    if recipe.backward:
        gy = rng.standard_normal(size=(B, T, C), dtype=np.float32)
        out["gy"], out["gy32"] = _store(gy, recipe.dtype)
    return out


def gate_input(shape, dtype: str, seed: int = 0, std: float = 2.0):
    """The receptance before its sigmoid, r ~ N(0, std^2) (std 2 reaches the
    saturated ends of the gate), as (storage array, exact float32 values).
    Drawn from its own stream so that the other inputs of a seed stay put."""
    rng = np.random.Generator(np.random.PCG64([seed, 0x5167]))
    r = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        r *= np.float32(std)
    return _store(r, dtype)


# ----------------------------------------------------------------------------
# RWKV-4 batched inference slots (web-rwkv "批量推理" / batched inference)
# ----------------------------------------------------------------------------

def wkv4_slot_inputs(S: int = 32, C: int = 4096, len_lo: int = 1, len_hi: int = 512,
                     dtype: str = "bf16", td_lo: float = -6.0, td_hi: float = 1.0,
                     u_lo: float = -1.0, u_hi: float = 1.0, seed: int = 0,
                     lengths: Optional[np.ndarray] = None) -> dict:
    """Draw S variable-length prompts for the slot-batched chunk step.

    Returns w, u [C] float32, ``lengths`` [S] int64 (~U{len_lo..len_hi} unless
    given), and for each slot its tokens packed back to back: k, v, k32, v32 of
    shape [sum(lengths), C], plus ``offsets`` [S+1] (prefix sums of lengths).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    td = rng.uniform(td_lo, td_hi, size=C)
    u = rng.uniform(u_lo, u_hi, size=C).astype(np.float32)
    if lengths is None:
        lengths = rng.integers(len_lo, len_hi + 1, size=S)
    lengths = np.asarray(lengths, dtype=np.int64)
    n = int(lengths.sum())
    k = rng.standard_normal(size=(n, C), dtype=np.float32)
    v = rng.standard_normal(size=(n, C), dtype=np.float32)
    out = {"w": np.exp(td).astype(np.float32), "u": u, "lengths": lengths,
           "offsets": np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)}
    out["k"], out["k32"] = _store(k, dtype)
    out["v"], out["v32"] = _store(v, dtype)
    return out


def feed_schedule(lengths, chunk: int):
    """Split each slot's prompt into calls of at most ``chunk`` tokens.

    Returns a list of calls; each call is an int64 array ``take[S]`` with the
    number of tokens slot s consumes in that call (0 = slot skipped), in order.
    Every slot gets min(remaining, chunk) tokens per call.
    """
    rem = np.asarray(lengths, dtype=np.int64).copy()
    calls = []
    while rem.sum() > 0:
        take = np.minimum(rem, chunk)
        calls.append(take.copy())
        rem -= take
    return calls


# ----------------------------------------------------------------------------
# RWKV-6 head-state recipes (rwkv-ops "rwkv6op 使用方法" / RWKV6_OP usage)
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Wkv6Recipe:
    name: str
    B: int
    T: int
    H: int
    K: int = 64
    d_mean: float = -1.0       # w = exp(-exp(d)), d ~ N(d_mean, d_std^2)
    d_std: float = 0.5
    u_lo: float = -1.0
    u_hi: float = 1.0

    def with_shape(self, B=None, T=None, H=None, name=None):
        return dataclasses.replace(
            self, B=self.B if B is None else B, T=self.T if T is None else T,
            H=self.H if H is None else H, name=name or self.name)


WKV6_RECIPES = {
    "wkv6_fwd_bf16_c2048": Wkv6Recipe("wkv6_fwd_bf16_c2048", 8, 4096, 32),
}


def wkv6_inputs(recipe: Wkv6Recipe, seed: int = 0) -> dict:
    """Draw one RWKV-6 workload: r, k, v, w as bf16 [B,T,H*K], u float32 [H*K].

    w = exp(-exp(d)) is evaluated in float64 and then rounded to bf16, so every
    stored decay lies in (0, 1]; ``w32`` is its exact float32 decoding.
    """
    B, T, HK = recipe.B, recipe.T, recipe.H * recipe.K
    rng = np.random.Generator(np.random.PCG64(seed))
    d = rng.standard_normal(size=(B, T, HK), dtype=np.float32)
    d = d.astype(np.float64) * recipe.d_std + recipe.d_mean
    w = np.exp(-np.exp(d)).astype(np.float32)
    del d
    u = rng.uniform(recipe.u_lo, recipe.u_hi, size=HK).astype(np.float32)
    out = {"u": u}
    out["w"], out["w32"] = _store(w, "bf16")
    del w
    for name in ("r", "k", "v"):
        x = rng.standard_normal(size=(B, T, HK), dtype=np.float32)
        out[name], out[name + "32"] = _store(x, "bf16")
    return out


# ----------------------------------------------------------------------------
# RWKV-7 (generalized delta rule) recipes
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Wkv7Recipe:
    name: str
    B: int
    T: int
    H: int
    K: int = 64
    d_mean: float = -1.0   # decay in log space w = -exp(d), d ~ N(d_mean, d_std^2)
    d_std: float = 0.5
    lr_lo: float = 0.0     # b = kappa * alpha with alpha ~ U(lr_lo, lr_hi) per (t, channel)
    lr_hi: float = 1.0

    def with_shape(self, B=None, T=None, H=None, name=None):
        return dataclasses.replace(
            self, B=self.B if B is None else B, T=self.T if T is None else T,
            H=self.H if H is None else H, name=name or self.name)


WKV7_RECIPES = {
    "wkv7_fwd_bf16_c2048": Wkv7Recipe("wkv7_fwd_bf16_c2048", 8, 4096, 32),
}


def wkv7_inputs(recipe: Wkv7Recipe, seed: int = 0) -> dict:
    """Draw one RWKV-7 workload: r, w, k, v, a, b as bf16 [B,T,H*K] (and their
    exact float32 decodings r32, ...). w = -exp(d) is the decay in log space;
    per (sample, token, head) a unit vector kappa is drawn (normalised
    N(0,1)), a = -kappa and b = kappa * alpha (the in-context removal and its
    rate, as in the delta rule); r, k, v ~ N(0,1). Draw order: d, kappa,
    alpha, r, k, v.
    """
    B, T, H, K = recipe.B, recipe.T, recipe.H, recipe.K
    HK = H * K
    rng = np.random.Generator(np.random.PCG64(seed))
    d = rng.standard_normal(size=(B, T, HK), dtype=np.float32).astype(np.float64) * recipe.d_std + recipe.d_mean
    out = {}
    out["w"], out["w32"] = _store((-np.exp(d)).astype(np.float32), "bf16")
    del d
    kap = rng.standard_normal(size=(B, T, H, K), dtype=np.float32).astype(np.float64)
    kap /= np.sqrt(np.sum(kap * kap, axis=-1, keepdims=True))
    kap = kap.reshape(B, T, HK)
    alpha = rng.uniform(recipe.lr_lo, recipe.lr_hi, size=(B, T, HK))
    out["a"], out["a32"] = _store((-kap).astype(np.float32), "bf16")
    out["b"], out["b32"] = _store((kap * alpha).astype(np.float32), "bf16")
    del kap, alpha
    for name in ("r", "k", "v"):
        x = rng.standard_normal(size=(B, T, HK), dtype=np.float32)
        out[name], out[name + "32"] = _store(x, "bf16")
    return out
