"""Counter-based, integer-exact bf16 fills (CPU side).

Definition (shared verbatim by the GPU fill kernel in ``synth/fill_gpu.cu``):

* ``key(seed, tensor) = SM(SM(seed) ^ tensor)`` where ``SM(s)`` is the first output of a
  SplitMix64 generator whose state is ``s`` (state += 0x9E3779B97F4A7C15, then the
  published output mix).
* Element ``e`` (row-major flat index) draws ``r_e = SM(key + e * 0x9E3779B97F4A7C15)``, i.e.
  the ``e``-th output of SplitMix64 seeded with ``key``.
* ``n_e = (sum of the four 16-bit lanes of r_e) - 131070``: an Irwin-Hall(4) variate on an
  integer grid, mean 0, variance ``4 * (65536^2 - 1) / 12``.  Exact in int32.
* ``value_e = bf16_rne(float32(n_e) * scale)`` with ``scale = float32(sigma / sd)``.  The
  integer converts to binary32 exactly and one IEEE multiply rounds once, so CPU and GPU
  agree bit for bit; no transcendental function is involved.

The distribution is a bounded (+-3.46 sigma) stand-in for N(0, sigma^2).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
IRWIN_HALL_SD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)


def _sm_mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_first(state: int) -> int:
    """First output of SplitMix64 seeded with ``state`` (python int in, python int out)."""
    with np.errstate(over="ignore"):
        z = np.array([state & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64) + GOLDEN
        return int(_sm_mix(z)[0])


def stream_key(seed: int, tensor: int) -> int:
    return splitmix64_first(splitmix64_first(seed) ^ (tensor & 0xFFFFFFFFFFFFFFFF))


def scale_for_sigma(sigma: float) -> np.float32:
    return np.float32(sigma / IRWIN_HALL_SD)


def float_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """binary32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_to_float(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _values_at(key: int, scale: np.float32, e: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = np.uint64(key) + e.astype(np.uint64) * GOLDEN + GOLDEN
        r = _sm_mix(z)
    mask = np.uint64(0xFFFF)
    s = (r & mask) + ((r >> np.uint64(16)) & mask) + ((r >> np.uint64(32)) & mask) + (r >> np.uint64(48))
    n = s.astype(np.int64) - 131070
    f = n.astype(np.float32) * np.float32(scale)
    return float_to_bf16_rne(f)


@dataclass(frozen=True)
class FillSpec:
    """One synthetic tensor: seed, tensor id within the seed, standard deviation."""
    seed: int
    tensor: int
    sigma: float

    @property
    def key(self) -> int:
        return stream_key(self.seed, self.tensor)

    @property
    def scale(self) -> np.float32:
        return scale_for_sigma(self.sigma)


def fill_bf16(spec: FillSpec, shape) -> np.ndarray:
    """Whole tensor as a uint16 (bf16 pattern) array of ``shape``, row-major."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    e = np.arange(n, dtype=np.uint64)
    return _values_at(spec.key, spec.scale, e).reshape(shape)


def fill_rows_bf16(spec: FillSpec, ncols: int, rows) -> np.ndarray:
    """Selected rows of a [*, ncols] tensor, regenerated without materialising the rest."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1)
    e = rows[:, None] * np.uint64(ncols) + np.arange(ncols, dtype=np.uint64)[None, :]
    return _values_at(spec.key, spec.scale, e.reshape(-1)).reshape(rows.size, ncols)


# ---------------------------------------------------------------------------------------
# FP8 (e4m3) tables.  Element e is the Irwin-Hall integer n_e above, encoded as the e4m3
# value nearest to n_e / 2^13 (ties to even, integer arithmetic only); the table's dequant
# scale is sigma * 2^13 / sd, so that dequantised values are ~ N(0, sigma^2) again.  The GPU
# generator in fill_gpu.cu runs the same integer steps.
FP8_FRAC_BITS = 13


def fp8_scale_for_sigma(sigma: float) -> np.float32:
    return np.float32(sigma * (1 << FP8_FRAC_BITS) / IRWIN_HALL_SD)


def encode_e4m3_int(n: np.ndarray) -> np.ndarray:
    """e4m3 code of n / 2^13 for integers |n| < 2^17 (round to nearest even)."""
    n = np.asarray(n, dtype=np.int64)
    a = np.abs(n)
    sign = (n < 0).astype(np.int64) << 7
    code = np.zeros_like(a)
    nz = a > 0
    msb = np.zeros_like(a)
    msb[nz] = np.floor(np.log2(a[nz])).astype(np.int64)
    # guard against log2 rounding at exact powers of two
    msb = np.where((a >> np.maximum(msb, 0)) >= 2, msb + 1, msb)
    msb = np.where((a >> np.maximum(msb, 0)) == 0, msb - 1, msb)
    e = msb - FP8_FRAC_BITS                      # a / 2^13 in [2^e, 2^(e+1))
    normal = nz & (e >= -6)
    # normal: keep 4 significant bits
    sh = np.maximum(msb - 3, 0)
    q = a >> sh
    rem = a - (q << sh)
    half = np.where(sh > 0, 1 << np.maximum(sh - 1, 0), 0)
    up = (sh > 0) & ((rem > half) | ((rem == half) & ((q & 1) == 1)))
    q = q + up
    e_n = np.where(q == 16, e + 1, e)
    q = np.where(q == 16, 8, q)
    code_n = ((e_n + 7) << 3) | (q - 8)
    # subnormal: value / 2^-9 = a / 16
    qs = a >> 4
    rs = a & 15
    ups = (rs > 8) | ((rs == 8) & ((qs & 1) == 1))
    code_s = qs + ups
    code = np.where(normal, code_n, np.where(nz, code_s, 0))
    return (code | np.where(nz, sign, 0)).astype(np.uint8)


def _fp8_at(key: int, e: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = np.uint64(key) + e.astype(np.uint64) * GOLDEN + GOLDEN
        r = _sm_mix(z)
    mask = np.uint64(0xFFFF)
    s = (r & mask) + ((r >> np.uint64(16)) & mask) + ((r >> np.uint64(32)) & mask) + (r >> np.uint64(48))
    return encode_e4m3_int(s.astype(np.int64) - 131070)


def fill_fp8(spec: FillSpec, shape) -> np.ndarray:
    shape = tuple(int(x) for x in shape)
    n = int(np.prod(shape))
    return _fp8_at(spec.key, np.arange(n, dtype=np.uint64)).reshape(shape)


def fill_rows_fp8(spec: FillSpec, ncols: int, rows) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1)
    e = rows[:, None] * np.uint64(ncols) + np.arange(ncols, dtype=np.uint64)[None, :]
    return _fp8_at(spec.key, e.reshape(-1)).reshape(rows.size, ncols)
