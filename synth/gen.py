"""Counter-based generator and value tables.

Every synthetic tensor is a set of *streams*. A stream is named by a 64-bit
key derived from (seed, kind, field...) and yields, at integer counter i, the
64-bit word ``mix64(key + i)``. The top 16 bits of that word index a
65536-entry table of values (normal quantiles for activations, uniform
quantiles for Xavier-uniform weights), so a value depends only on
(seed, kind, fields, counter), never on buffer shapes or on which device
produced it. The CUDA fill library in ``synth/csrc`` implements the same
definition with integer arithmetic and the same uploaded table, so the bytes
it writes are bit-identical to the ones produced here.

``mix64`` is the SplitMix64 output function (G. Steele, D. Lea, C. Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014): add the golden
gamma 0x9E3779B97F4A7C15, then two xor-shift-multiply rounds and a final
xor-shift.
"""

from __future__ import annotations

import numpy as np
from scipy.special import ndtri

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MUL1 = 0xBF58476D1CE4E5B9
MUL2 = 0x94D049BB133111EB

# Stream kinds. Fields after the kind are listed per kind.
KIND_KV = 1      # (layer, row, kv_head, k_or_v); counter = (position-1)*d + dim
KIND_Q = 2       # (layer, row, q_head);         counter = step*d + dim
KIND_HIDDEN = 3  # (which, row) which: 0 h_{t-1}, 1 E(x_t), 2 h^L_t; counter = step*H + j
KIND_W1 = 4      # (0,);                          counter = m*in_dim + k
KIND_VEC = 5     # (which,) small vectors: 0 = w2; counter = m
KIND_NEEDLE = 6  # (layer, row);                  counter = dim (needle direction)

TABLE_BITS = 16
TABLE_SIZE = 1 << TABLE_BITS


def mix64_int(x: int) -> int:
    """SplitMix64 output function on a Python int (wrapping mod 2**64)."""
    z = (x + GAMMA) & MASK64
    z = ((z ^ (z >> 30)) * MUL1) & MASK64
    z = ((z ^ (z >> 27)) * MUL2) & MASK64
    return z ^ (z >> 31)


def mix64(x: np.ndarray) -> np.ndarray:
    """Vectorised SplitMix64 output function on a uint64 array (new array)."""
    z = np.asarray(x, dtype=np.uint64).copy()
    with np.errstate(over="ignore"):
        z += np.uint64(GAMMA)
        t = z >> np.uint64(30)
        z ^= t
        z *= np.uint64(MUL1)
        t = z >> np.uint64(27)
        z ^= t
        z *= np.uint64(MUL2)
        t = z >> np.uint64(31)
        z ^= t
    return z


def stream_key(seed: int, kind: int, *fields: int) -> int:
    """Key of one stream: fold (seed, kind, fields...) through mix64."""
    k = mix64_int(seed & MASK64)
    k = mix64_int(k ^ (kind & MASK64))
    for f in fields:
        k = mix64_int(k ^ (int(f) & MASK64))
    return k


# --------------------------------------------------------------------------
# bf16 helpers (round-to-nearest-even), used to materialise generated values
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    r = r.astype(np.uint32).astype(np.uint16)
    if nan.any():
        r = np.where(nan, np.uint16(0x7FC0), r)
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float64/float32 -> float32 (RNE) -> bf16 bits (RNE)."""
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32))


# --------------------------------------------------------------------------
# value tables
# --------------------------------------------------------------------------

def normal_table(sigma: float, dtype: str) -> np.ndarray:
    """65536 quantiles of N(0, sigma^2) at the cell midpoints (i+0.5)/65536.

    dtype "bf16" returns uint16 bit patterns, "f32" returns float32.
    """
    p = (np.arange(TABLE_SIZE, dtype=np.float64) + 0.5) / TABLE_SIZE
    z = ndtri(p) * float(sigma)
    return _materialise(z, dtype)


def uniform_table(bound: float, dtype: str) -> np.ndarray:
    """65536 quantiles of U(-bound, bound) at the cell midpoints."""
    p = (np.arange(TABLE_SIZE, dtype=np.float64) + 0.5) / TABLE_SIZE
    z = (2.0 * p - 1.0) * float(bound)
    return _materialise(z, dtype)


def _materialise(z: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_round_bits(z)
    if dtype == "f32":
        return z.astype(np.float32)
    raise ValueError(f"unsupported dtype {dtype!r}")


def table_index(key: int, counters: np.ndarray) -> np.ndarray:
    """Top 16 bits of mix64(key + counter) for an array of counters."""
    with np.errstate(over="ignore"):
        c = np.asarray(counters, dtype=np.uint64) + np.uint64(key)
    return (mix64(c) >> np.uint64(64 - TABLE_BITS)).astype(np.int64)


def table_values(key: int, start: int, count: int, table: np.ndarray) -> np.ndarray:
    """Values of one stream at counters start .. start+count-1."""
    c = np.arange(count, dtype=np.uint64) + np.uint64(start)
    return table[table_index(key, c)]


def fill_streams(keys, offsets, n_outer: int, inner: int, table: np.ndarray) -> np.ndarray:
    """Array [n_outer][n_streams][inner] with
    out[i, s, j] = table[top16(mix64(keys[s] + offsets[s] + i*inner + j))].

    This is the exact definition the CUDA fill kernel implements.
    """
    keys = np.asarray(keys, dtype=np.uint64).reshape(-1)
    offs = np.asarray(offsets, dtype=np.uint64).reshape(-1)
    ns = keys.shape[0]
    out = np.empty((n_outer, ns, inner), dtype=table.dtype)
    c = (np.arange(n_outer, dtype=np.uint64)[:, None] * np.uint64(inner)
         + np.arange(inner, dtype=np.uint64)[None, :])
    for s in range(ns):
        with np.errstate(over="ignore"):
            cs = c + np.uint64(int(offs[s]))
        out[:, s, :] = table[table_index(int(keys[s]), cs)]
    return out
