"""Seeded synthetic inputs for the five kernelized-linear-attention workloads.

This module draws random numbers and rounds them to the storage dtype. It holds
none of the method's arithmetic (no feature map, no state, no attention), so both
the CUDA path and the fp64 oracle can be fed from it.

Recipes (all use NumPy's PCG64 ``default_rng(seed)``):

* ``normal``: q, k, v drawn in that order, each a full C-order tensor of iid
  N(0, 1/d) values (standard normal draws scaled by d**-0.5).
* ``unit_qk``: q and k rows are standard normal vectors normalised to unit L2
  length and then scaled by d**-0.5; v is iid N(0, 1).
* ``recall``: the associative-recall shape used for the LoLA sparse-cache
  workload. A pool of 512 standard normal vectors normalised to unit length is
  drawn first. For each head, position 0 takes a uniform pool index; every later
  position t copies the pool index of a uniformly chosen earlier position with
  probability 0.3 and otherwise draws a fresh uniform pool index. Keys are the
  pool vectors at those indices. The query at position t is the key at a
  uniformly chosen position u in [0, t] (a recall query). v is iid N(0, 1).

Large tensors (above ``_F64_LIMIT`` elements) are drawn directly in float32 to
keep host memory bounded; the seed still fixes every value. Values are rounded
to the storage dtype once (fp64 -> fp32 -> bf16, round to nearest even), and
every consumer reads those rounded values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

_F64_LIMIT = 1 << 24

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "prefill", "decode" or "lola"
    B: int
    H: int
    d: int
    T: int = 0
    chunk: int = 64
    dtype: str = "bf16"
    eps: float = 1e-6
    seed: int = 0
    recipe: str = "normal"
    prefix: int = 0
    steps: int = 0
    window: int = 0
    cache: int = 0
    pool: int = 512
    repeat: float = 0.3
    extra: dict = field(default_factory=dict)

    @property
    def D(self) -> int:
        return self.d * (self.d + 1) // 2


WORKLOADS = {
    w.name: w
    for w in [
        Workload("pr1_ref_t256_d16", "prefill", B=1, H=1, T=256, d=16, chunk=64,
                 dtype="f32", seed=0, recipe="normal"),
        Workload("prefill_b4_h8_t2048_d32", "prefill", B=4, H=8, T=2048, d=32, chunk=64,
                 dtype="bf16", seed=1, recipe="normal"),
        Workload("long_prefill_b2_h16_t16384_d64", "prefill", B=2, H=16, T=16384, d=64,
                 chunk=128, dtype="bf16", seed=2, recipe="unit_qk"),
        Workload("decode_b64_h16_d64", "decode", B=64, H=16, d=64, prefix=4096, steps=256,
                 dtype="bf16", seed=3, recipe="normal"),
        Workload("lola_b2_h8_t8192_d64", "lola", B=2, H=8, T=8192, d=64, window=64,
                 cache=128, dtype="bf16", seed=4, recipe="recall"),
    ]
}


def _normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    if n > _F64_LIMIT:
        x = rng.standard_normal(shape, dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        return x
    x = rng.standard_normal(shape)
    if scale != 1.0:
        x *= scale
    return x


def _unit_rows(x: np.ndarray) -> np.ndarray:
    nrm = np.sqrt(np.sum(np.asarray(x, dtype=np.float64) ** 2, axis=-1, keepdims=True))
    return (x / nrm).astype(x.dtype, copy=False)


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round to the storage dtype once: fp64 -> fp32 -> (bf16, nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(DTYPES[dtype]).contiguous()


def prefill_inputs(B: int, H: int, T: int, d: int, dtype: str = "bf16", seed: int = 0,
                   recipe: str = "normal"):
    """q, k, v as CPU tensors of shape [B, H, T, d] in the storage dtype."""
    rng = np.random.default_rng(seed)
    shape = (B, H, T, d)
    if recipe == "normal":
        q = _normal(rng, shape, d ** -0.5)
        k = _normal(rng, shape, d ** -0.5)
        v = _normal(rng, shape, d ** -0.5)
    elif recipe == "unit_qk":
        q = _unit_rows(_normal(rng, shape)) * (d ** -0.5)
        k = _unit_rows(_normal(rng, shape)) * (d ** -0.5)
        v = _normal(rng, shape)
    elif recipe == "recall":
        return recall_inputs(B, H, T, d, dtype=dtype, seed=seed)
    else:
        raise ValueError(f"unknown recipe {recipe!r}")
    return to_storage(q, dtype), to_storage(k, dtype), to_storage(v, dtype)


def recall_inputs(B: int, H: int, T: int, d: int, dtype: str = "bf16", seed: int = 4,
                  pool: int = 512, repeat: float = 0.3):
    """Associative-recall keys/queries from a unit-vector pool (see module docstring)."""
    rng = np.random.default_rng(seed)
    P = _unit_rows(rng.standard_normal((pool, d)))
    q = np.empty((B, H, T, d))
    k = np.empty((B, H, T, d))
    for b in range(B):
        for h in range(H):
            coin = rng.random(T)
            fresh = rng.integers(0, pool, size=T)
            back = rng.random(T)
            qpick = rng.random(T)
            idx = np.empty(T, dtype=np.int64)
            idx[0] = fresh[0]
            for t in range(1, T):
                if coin[t] < repeat:
                    idx[t] = idx[int(back[t] * t)]
                else:
                    idx[t] = fresh[t]
            k[b, h] = P[idx]
            u = np.minimum((qpick * (np.arange(T) + 1)).astype(np.int64), np.arange(T))
            q[b, h] = P[idx[u]]
    v = rng.standard_normal((B, H, T, d))
    return to_storage(q, dtype), to_storage(k, dtype), to_storage(v, dtype)


def decode_inputs(B: int, H: int, d: int, prefix: int, steps: int, dtype: str = "bf16",
                  seed: int = 3):
    """Prefix keys/values [B, H, prefix, d] and per-step q, k, v [steps, B, H, d]."""
    rng = np.random.default_rng(seed)
    kp = _normal(rng, (B, H, prefix, d), d ** -0.5)
    vp = _normal(rng, (B, H, prefix, d), d ** -0.5)
    q = _normal(rng, (steps, B, H, d), d ** -0.5)
    k = _normal(rng, (steps, B, H, d), d ** -0.5)
    v = _normal(rng, (steps, B, H, d), d ** -0.5)
    return tuple(to_storage(x, dtype) for x in (kp, vp, q, k, v))


def candidate_inputs(B: int, H: int, n: int, d: int, dtype: str = "bf16", seed: int = 5,
                     ties: bool = False):
    """SRE candidates: k, v [B, H, n, d] and strictly increasing positions [B, H, n].

    With ``ties`` every other candidate repeats its predecessor's key and value,
    so equal scores occur on purpose.
    """
    rng = np.random.default_rng(seed)
    k = _normal(rng, (B, H, n, d), d ** -0.5)
    v = _normal(rng, (B, H, n, d), d ** -0.5)
    if ties:
        m = n // 2
        k[:, :, 1:2 * m:2] = k[:, :, 0:2 * m:2]
        v[:, :, 1:2 * m:2] = v[:, :, 0:2 * m:2]
    gaps = rng.integers(1, 4, size=(B, H, n))
    pos = np.cumsum(gaps, axis=-1).astype(np.int32)
    return to_storage(k, dtype), to_storage(v, dtype), torch.from_numpy(pos)


def state_inputs(B: int, H: int, d: int, tokens: int, seed: int = 6):
    """Keys/values whose rank-one sums build a state: [B, H, tokens, d] fp32."""
    rng = np.random.default_rng(seed)
    k = _normal(rng, (B, H, tokens, d), d ** -0.5)
    v = _normal(rng, (B, H, tokens, d), d ** -0.5)
    return to_storage(k, "f32"), to_storage(v, "f32")
