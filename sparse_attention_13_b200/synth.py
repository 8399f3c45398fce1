"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module holds no arithmetic of the method.  It defines one counter-based
generator and draws every element of every input tensor from it, so the host
(numpy) and the device (a small CUDA kernel in ``libdsa_synth.so``) produce
bit-identical tensors from (seed, kind, layer, element index) alone.  The oracle
never imports this module; tests hand the same arrays to both sides.

Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014): output n of a stream with key
``x`` is ``mix64(x + (n + 1) * GAMMA)``.  Each (seed, kind, layer) gets its own
key ``mix64(seed * GAMMA + kind * 2**40 + layer * 2**24 + 1)``.

Distributions (element value from one 64-bit draw ``z``):
  INT9   integer uniform in [-4, 4]: ((z >> 32) * 9 >> 32) - 4   (exact in bf16)
  POW2W  +-2**-m, m uniform in {0..3}: sign = bit 63, m = bits 61..62
  NORMAL sigma * (sum of the four 16-bit lanes of z - 131070) / std, computed
         as one fp32 multiply of an exact integer (Irwin-Hall(4): a bounded,
         normal-shaped law; identical on host and device), rounded to bf16 by
         round-to-nearest-even when the tensor is bf16.
Layer correlation (``corr=True``): layer l's value is x_l = 0.9 x_{l-1} +
0.44 n_l with n_l drawn like layer 0, evaluated in fp32 with separate
round-to-nearest multiplies and add; bf16 tensors round x_l to bf16, INT9
tensors round half-to-even and clamp to [-4, 4].
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)

INT9, POW2W, NORMAL = 0, 1, 2

# tensor kinds (stream ids)
Q_IDX, K_IDX, W, Q, KV, K_SEP, V_SEP = 1, 2, 3, 4, 5, 6, 7

_IH_STD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)


def normal_scale(sigma: float) -> np.float32:
    return np.float32(sigma / _IH_STD)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * M1
    z = z ^ (z >> np.uint64(27))
    z = z * M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, kind: int, layer: int) -> np.uint64:
    with np.errstate(over="ignore"):
        x = (np.uint64(seed) * GAMMA + np.uint64(kind << 40) + np.uint64(layer << 24)
             + np.uint64(1))
        return _mix64(np.array([x], dtype=np.uint64))[0]


def raw(seed: int, kind: int, layer: int, index: np.ndarray) -> np.ndarray:
    key = stream_key(seed, kind, layer)
    n = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + (n + np.uint64(1)) * GAMMA)


def _draw(z: np.ndarray, dist: int, c: np.float32) -> np.ndarray:
    if dist == INT9:
        return ((((z >> np.uint64(32)) * np.uint64(9)) >> np.uint64(32)).astype(np.int64) - 4).astype(np.float32)
    if dist == POW2W:
        sign = np.where((z >> np.uint64(63)) == 1, np.float32(-1.0), np.float32(1.0))
        m = ((z >> np.uint64(61)) & np.uint64(3)).astype(np.int32)
        return (sign * np.ldexp(np.float32(1.0), -m).astype(np.float32)).astype(np.float32)
    if dist == NORMAL:
        s = np.zeros(z.shape, dtype=np.int64)
        for i in range(4):
            s += ((z >> np.uint64(16 * i)) & np.uint64(0xFFFF)).astype(np.int64)
        return (s - 131070).astype(np.float32) * np.float32(c)
    raise ValueError(dist)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def values(seed: int, kind: int, dist: int, layer: int, index, *, sigma: float = 1.0,
           corr: bool = False, bf16: bool = True) -> np.ndarray:
    """Element values at flat ``index`` of tensor (seed, kind, layer).

    Returns uint16 bf16 bits when ``bf16`` else float32."""
    index = np.asarray(index, dtype=np.uint64)
    c = normal_scale(sigma)
    layers = range(layer + 1) if corr else [layer]
    x = None
    for l in layers:
        v = _draw(raw(seed, kind, l, index), dist, c)
        if x is None:
            x = v
        else:
            x = (np.float32(0.9) * x) + (np.float32(0.44) * v)
        if dist == INT9:
            x = np.clip(np.rint(x), -4, 4).astype(np.float32)
        elif bf16:
            x = bf16_bits_to_f32(f32_to_bf16_bits(x))
    return f32_to_bf16_bits(x) if bf16 else x.astype(np.float32)


def tensor(seed: int, kind: int, dist: int, layer: int, shape, **kw) -> np.ndarray:
    n = int(np.prod(shape))
    return values(seed, kind, dist, layer, np.arange(n, dtype=np.uint64), **kw).reshape(shape)


def rows(seed: int, kind: int, dist: int, layer: int, shape, row_ids, **kw) -> np.ndarray:
    """Selected rows (along the flattened leading dims) of a tensor whose
    trailing dimension is ``shape[-1]``; lets the oracle read slices of tensors
    too large for the host."""
    inner = int(shape[-1])
    row_ids = np.asarray(row_ids, dtype=np.uint64).reshape(-1, 1)
    idx = row_ids * np.uint64(inner) + np.arange(inner, dtype=np.uint64)[None, :]
    return values(seed, kind, dist, layer, idx, **kw)


# ---------------------------------------------------------------------------
# device generator (same definition, CUDA kernel in libdsa_synth.so)
_synth = None


def _synth_lib():
    global _synth
    if _synth is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa_synth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        lib.dsa_synth_fill.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_uint64, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_void_p]
        lib.dsa_synth_fill.restype = ctypes.c_int
        _synth = lib
    return _synth


def fill_cuda(t, seed: int, kind: int, dist: int, layer: int, *, sigma: float = 1.0,
              corr: bool = False, start: int = 0) -> None:
    """Fill a contiguous CUDA tensor (bf16 or float32) with the elements
    [start, start + t.numel()) of tensor (seed, kind, layer)."""
    import torch
    assert t.is_cuda and t.is_contiguous()
    is_bf16 = t.dtype == torch.bfloat16
    assert is_bf16 or t.dtype == torch.float32
    stream = torch.cuda.current_stream(t.device).cuda_stream
    rc = _synth_lib().dsa_synth_fill(
        ctypes.c_void_p(t.data_ptr()), t.numel(), start, seed, kind, dist, layer,
        float(normal_scale(sigma)), int(corr), int(is_bf16), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"dsa_synth_fill failed: {rc}")
